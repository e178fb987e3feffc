// Router GEMV, top-k softmax and the expert-grouped permutation of the
// (token, rank) pairs, all on the device.
//
// turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs: the caller's M
// router GEMVs produce fp32 logits; the reference then reads them back and runs
// router_topk_gemma4 per token on the host, and next_routed_sub_batch /
// encode_routes build the routes in PAIR order (token-major, rank within) with
// fp16 routing weights. Here none of it leaves the GPU: one kernel computes the
// logits (plus the shared-expert gate logit), a single-CTA kernel selects the
// top-k, computes the weights and builds the grouped permutation.
#include <algorithm>

#include "launch.cuh"
#include "norm.cuh"
#include "route.cuh"

namespace moeffn {

namespace {

constexpr int kRouterThreads = 128;

// logits[t][e] = Wr[e] . x[t] (fp32 accumulate), one CTA per (token, row);
// row e == E is the shared expert gate vector (bf16), written to gate_logit[t].
__global__ void __launch_bounds__(kRouterThreads) k_router_logits(const RouterArgs a) {
  __shared__ float red[kRouterThreads / 32];
  __shared__ float s_inv;
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  const int e = blockIdx.y;
  if (a.route_cnt != nullptr && t == 0 && e == 0 && threadIdx.x == 0) *a.route_cnt = 0;   // for the top-k kernel next
  const bool gate_row = (e == a.E);
  const uint16_t* x = a.x + (size_t)t * a.H;
  const bool norm = a.norm_w != nullptr;
  float inv = 0.f;
  if (norm) {
    // Input norm folded in: every CTA of the token finds the row's inv_rms
    // (the row is a few KB); the CTA of expert 0 also stores m.
    float ss = warp_sum(row_sumsq_part(x, a.H, threadIdx.x, kRouterThreads));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      float v = 0.f;
      for (int i = 0; i < kRouterThreads / 32; ++i) v += red[i];   // fixed order
      s_inv = inv_rms_of(v, a.H, a.eps);
    }
    __syncthreads();
    inv = s_inv;
    if (e == 0)
      for (int k = threadIdx.x; k < a.H; k += kRouterThreads)
        a.m_out[(size_t)t * a.H + k] = prenorm_elem(x[k], a.norm_w[k], inv);
  }
  // The token row's k-th value as the layer's input m (normalized or given).
  auto xval = [&](uint32_t bits16, int k) -> float {
    return norm ? bf16_bits_to_float(prenorm_elem((uint16_t)bits16, a.norm_w[k], inv))
                : bf16_bits_to_float((uint16_t)bits16);
  };
  float acc = 0.f;
  if (!gate_row && a.router_f32) {
    const float* w = reinterpret_cast<const float*>(a.router) + (size_t)e * a.H;
    for (int k = threadIdx.x * 4; k < a.H; k += kRouterThreads * 4) {
      const float4 wv = *reinterpret_cast<const float4*>(w + k);
      const uint2 xv = *reinterpret_cast<const uint2*>(x + k);
      acc = fmaf(wv.x, xval(xv.x & 0xFFFFu, k), acc);
      acc = fmaf(wv.y, xval(xv.x >> 16, k + 1), acc);
      acc = fmaf(wv.z, xval(xv.y & 0xFFFFu, k + 2), acc);
      acc = fmaf(wv.w, xval(xv.y >> 16, k + 3), acc);
    }
  } else {
    const uint16_t* w = gate_row ? a.w_sg : reinterpret_cast<const uint16_t*>(a.router) + (size_t)e * a.H;
    for (int k = threadIdx.x * 8; k < a.H; k += kRouterThreads * 8) {
      const uint4 wv = *reinterpret_cast<const uint4*>(w + k);
      const uint4 xv = *reinterpret_cast<const uint4*>(x + k);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc = fmaf(__uint_as_float(ww[j] << 16), xval(xx[j] & 0xFFFFu, k + 2 * j), acc);
        acc = fmaf(__uint_as_float(ww[j] & 0xFFFF0000u), xval(xx[j] >> 16, k + 2 * j + 1), acc);
      }
    }
  }
  acc = warp_sum(acc);
  __syncthreads();   // red is reused
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int i = 0; i < kRouterThreads / 32; ++i) v += red[i];   // fixed order
    if (gate_row) a.gate_logit[t] = v;
    else a.logits[(size_t)t * a.E + e] = v;
  }
}

// m = rms_norm(x, w) of one row per CTA.
__global__ void __launch_bounds__(256) k_prenorm_rows(const PrenormArgs a) {
  __shared__ float red[8];
  __shared__ float s_inv;
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  const uint16_t* x = a.x + (size_t)t * a.H;
  const float ss = warp_sum(row_sumsq_part(x, a.H, threadIdx.x, 256));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int i = 0; i < 8; ++i) v += red[i];   // fixed order
    s_inv = inv_rms_of(v, a.H, a.eps);
  }
  __syncthreads();
  const float inv = s_inv;
  for (int k = threadIdx.x; k < a.H; k += 256) a.m[(size_t)t * a.H + k] = prenorm_elem(x[k], a.w[k], inv);
}

// (value, index) order of the top-k: larger value first, lower index on ties.
__device__ __forceinline__ bool beats(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Top-k of one token by one warp: every lane holds up to PL logits (experts
// lane, lane+32, ...) of the token's row `l`; k rounds of a warp-wide
// arg-max, the winner's lane retires it. Weights: softmax over the k selected
// logits times the per-expert scale of the selected expert (ones unless
// given), rounded to fp16. The experts also go to sidx (shared memory), if given.
template <int PL>
__device__ __forceinline__ void topk_token(const RouteArgs& a, const float* l, int t, int lane, int* sidx) {
  float lv[PL];
  unsigned taken = 0;
#pragma unroll
  for (int j = 0; j < PL; ++j) {
    const int e = lane + 32 * j;
    lv[j] = e < a.E ? l[e] : 0.f;
  }
  float top0 = 0.f, zsum = 0.f;
  float zr[kMaxTopK];
  int ir[kMaxTopK];
  for (int r = 0; r < a.k; ++r) {
    float bv = -INFINITY;   // lanes without a candidate never win
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < PL; ++j) {
      const int e = lane + 32 * j;
      if (e < a.E && !((taken >> j) & 1u) && beats(lv[j], e, bv, bi)) {
        bv = lv[j];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (beats(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (r == 0) top0 = bv;
    zr[r] = expf(bv - top0);
    ir[r] = bi;
    zsum += zr[r];
  }
  if (lane < a.k) {   // lane r stores rank r
    float z = 0.f;
    int e = 0;
    for (int r = 0; r < a.k; ++r)
      if (r == lane) { z = zr[r]; e = ir[r]; }
    const float sc = a.scale != nullptr ? a.scale[e] : 1.0f;
    a.idx[t * a.k + lane] = e;
    a.w[t * a.k + lane] = __half2float(__float2half_rn(z / zsum * sc));
    if (sidx != nullptr) sidx[t * a.k + lane] = e;
  }
}

// Experts up to which placement runs with a per-warp count table.
constexpr int kWarpTableE = 128;
constexpr int kRouteWarps = 8;   // tokens (warps) per top-k CTA

// Shared memory of the placing CTA (ints): counts, running, offsets and the
// per-warp count table.
__host__ __device__ inline size_t route_smem_ints(int E) {
  return (size_t)(3 * E + 1) + (E <= kWarpTableE ? (size_t)kRouteWarps * E : 0);
}

// The stable expert-grouped order of the pairs p = t*k + r, by one CTA:
// warp-aggregated counts, offsets and union, then the placement chunk by
// chunk of the block's threads -- a pair's position is its expert's offset,
// plus the pairs of that expert in earlier chunks, in earlier warps of the
// chunk (a per-warp count table with a prefix over warps) and in earlier
// lanes of its warp (match_any). Experts come from global memory (written by
// other CTAs: read through L2).
__device__ void place_pairs(const RouteArgs& a, int* sm) {
  const int E = a.E, P = a.M * a.k;
  const bool table = E <= kWarpTableE;
  int* counts = sm;                                   // [E]
  int* running = counts + E;                          // [E]
  int* offs = running + E;                            // [E+1]
  int* wc = offs + E + 1;                             // [kRouteWarps][E] (table)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) { counts[e] = 0; running[e] = 0; }
  __syncthreads();
  for (int base = warp * 32; base < P; base += nwarps * 32) {   // warp-aggregated counts
    const int p = base + lane;
    const bool act = p < P;
    const unsigned active = __ballot_sync(0xffffffffu, act);
    if (act) {
      const int e = __ldcg(a.idx + p);
      const unsigned same = __match_any_sync(active, e);
      if ((same & ((1u << lane) - 1u)) == 0) atomicAdd(&counts[e], __popc(same));
    }
  }
  __syncthreads();
  if (warp == 0) {
    // Exclusive prefix of the counts and the ascending union, 32 experts at a
    // time: a warp scan of the counts and a ballot of the nonzero ones.
    int acc = 0, nu = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int cnt = e < E ? counts[e] : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < E) offs[e] = acc + incl - cnt;
      const unsigned nz = __ballot_sync(0xffffffffu, cnt > 0);
      if (cnt > 0 && a.union_list != nullptr) a.union_list[nu + __popc(nz & ((1u << lane) - 1u))] = e;
      acc += __shfl_sync(0xffffffffu, incl, 31);
      nu += __popc(nz);
    }
    if (lane == 0) {
      offs[E] = acc;
      if (a.n_union != nullptr) *a.n_union = nu;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) a.offsets[e] = offs[e];
  if (table) {
    for (int base = 0; base < P; base += blockDim.x) {
      for (int i = threadIdx.x; i < nwarps * E; i += blockDim.x) wc[i] = 0;
      __syncthreads();
      const int p = base + threadIdx.x;
      const bool act = p < P;
      const unsigned active = __ballot_sync(0xffffffffu, act);
      int e = 0, rank = 0;
      if (act) {
        e = __ldcg(a.idx + p);
        const unsigned same = __match_any_sync(active, e);
        rank = __popc(same & ((1u << lane) - 1u));
        if (rank == 0) wc[warp * E + e] = __popc(same);
      }
      __syncthreads();
      for (int e2 = threadIdx.x; e2 < E; e2 += blockDim.x) {   // exclusive prefix over warps
        int s = running[e2];
        for (int w = 0; w < nwarps; ++w) {
          const int c = wc[w * E + e2];
          wc[w * E + e2] = s;
          s += c;
        }
        running[e2] = s;
      }
      __syncthreads();
      if (act) {
        const int pos = offs[e] + wc[warp * E + e] + rank;
        a.perm[pos] = p;
        if (a.inv != nullptr) a.inv[p] = pos;
      }
      __syncthreads();
    }
  } else if (threadIdx.x < 32) {
    // Many experts: warp 0 walks the pairs in order, 32 at a time; equal
    // experts inside a chunk are ranked by lane (match_any + popc).
    for (int base = 0; base < P; base += 32) {
      const int p = base + lane;
      const bool act = p < P;
      const unsigned active = __ballot_sync(0xffffffffu, act);
      if (act) {
        const int e = __ldcg(a.idx + p);
        const unsigned same = __match_any_sync(active, e);
        const int rank = __popc(same & ((1u << lane) - 1u));
        const int pos = offs[e] + running[e] + rank;
        a.perm[pos] = p;
        if (a.inv != nullptr) a.inv[p] = pos;
        __syncwarp(active);
        if (rank == 0) running[e] += __popc(same);
      }
      __syncwarp();
    }
  }
}

// Top-k of kRouteWarps tokens per CTA (a warp each); the last CTA to finish
// (an arrival counter, zeroed by the kernel that runs before: the router, or
// the caller) places the pairs of all tokens.
template <int PL>
__global__ void __launch_bounds__(32 * kRouteWarps) k_route(const RouteArgs a) {
  extern __shared__ int sm[];
  __shared__ int s_last;
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + warp;
  if (t < a.M) topk_token<PL>(a, a.logits + (size_t)t * a.E, t, lane, nullptr);
  if (a.perm == nullptr) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(a.counter, 1);
    s_last = old == (int)gridDim.x - 1;
    if (s_last) *a.counter = 0;   // ready for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  place_pairs(a, sm);
}

// Token rows in expert-grouped pair order: the B operand rows of the grouped
// expert GEMMs. One CTA per slot, 16-byte copies.
__global__ void __launch_bounds__(128) k_gather_rows(const GatherArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int s = blockIdx.x;
  const int t = a.perm[s] / a.topk;
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
  uint4* dst = reinterpret_cast<uint4*>(a.xg + (size_t)s * a.H);
  for (int i = threadIdx.x; i < a.H / 8; i += blockDim.x) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_prenorm_rows(const PrenormArgs& a, cudaStream_t s) {
  return launch_pdl(k_prenorm_rows, dim3(a.M), dim3(256), 0, s, a);
}

cudaError_t launch_gather_rows(const GatherArgs& a, cudaStream_t s) {
  return launch_pdl(k_gather_rows, dim3(a.P), dim3(128), 0, s, a);
}

cudaError_t launch_router_logits(const RouterArgs& a, cudaStream_t s) {
  const int rows = a.E + (a.w_sg != nullptr ? 1 : 0);
  return launch_pdl(k_router_logits, dim3(a.M, rows), dim3(kRouterThreads), 0, s, a);
}

namespace {
template <int PL>
cudaError_t launch_route_t(const RouteArgs& a, cudaStream_t s) {
  const size_t smem = route_smem_ints(a.E) * sizeof(int);
  if (a.perm != nullptr && a.counter == nullptr) return cudaErrorInvalidValue;
  const int blocks = (a.M + kRouteWarps - 1) / kRouteWarps;
  return launch_pdl(k_route<PL>, dim3(blocks), dim3(32 * kRouteWarps), smem, s, a);
}
}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  const int pl = (a.E + 31) / 32;
  if (pl <= 1) return launch_route_t<1>(a, s);
  if (pl <= 2) return launch_route_t<2>(a, s);
  if (pl <= 4) return launch_route_t<4>(a, s);
  if (pl <= 8) return launch_route_t<8>(a, s);
  return launch_route_t<32>(a, s);
}

}  // namespace moeffn
