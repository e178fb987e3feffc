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
#include "route.cuh"

namespace moeffn {

namespace {

constexpr int kRouterWarps = 8;

// logits[t][e] = Wr[e] . x[t] (fp32 accumulate); row e == E is the shared
// expert gate vector (bf16), written to gate_logit[t].
__global__ void __launch_bounds__(kRouterWarps * 32) k_router_logits(const RouterArgs a) {
  const int t = blockIdx.x;
  const int e = blockIdx.y * kRouterWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int rows = a.E + (a.w_sg != nullptr ? 1 : 0);
  if (e >= rows) return;
  const uint16_t* x = a.x + (size_t)t * a.H;
  float acc = 0.f;
  const bool gate_row = (e == a.E);
  if (!gate_row && a.router_f32) {
    const float* w = reinterpret_cast<const float*>(a.router) + (size_t)e * a.H;
    for (int k = lane * 4; k < a.H; k += 128) {
      const float4 wv = *reinterpret_cast<const float4*>(w + k);
      const uint2 xv = *reinterpret_cast<const uint2*>(x + k);
      acc = fmaf(wv.x, __uint_as_float(xv.x << 16), acc);
      acc = fmaf(wv.y, __uint_as_float(xv.x & 0xFFFF0000u), acc);
      acc = fmaf(wv.z, __uint_as_float(xv.y << 16), acc);
      acc = fmaf(wv.w, __uint_as_float(xv.y & 0xFFFF0000u), acc);
    }
  } else {
    const uint16_t* w = gate_row ? a.w_sg : reinterpret_cast<const uint16_t*>(a.router) + (size_t)e * a.H;
    for (int k = lane * 8; k < a.H; k += 256) {
      const uint4 wv = *reinterpret_cast<const uint4*>(w + k);
      const uint4 xv = *reinterpret_cast<const uint4*>(x + k);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc = fmaf(__uint_as_float(ww[j] << 16), __uint_as_float(xx[j] << 16), acc);
        acc = fmaf(__uint_as_float(ww[j] & 0xFFFF0000u), __uint_as_float(xx[j] & 0xFFFF0000u), acc);
      }
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    if (gate_row) a.gate_logit[t] = acc;
    else a.logits[(size_t)t * a.E + e] = acc;
  }
}

// One CTA: per token the k largest logits ordered by (logit desc, index asc),
// softmax over them times the per-expert scale (ones), rounded to fp16; then
// the stable expert-grouped order of the pairs p = t*k + r.
__global__ void __launch_bounds__(1024) k_route(const RouteArgs a) {
  extern __shared__ int sm[];
  int* counts = sm;                 // [E]
  int* running = sm + a.E;          // [E]
  int* offs = sm + 2 * a.E;         // [E+1]
  const int P = a.M * a.k;

  for (int t = threadIdx.x; t < a.M; t += blockDim.x) {
    const float* l = a.logits + (size_t)t * a.E;
    int chosen[kMaxTopK];
    float val[kMaxTopK];
    for (int r = 0; r < a.k; ++r) {
      int best = -1;
      float bv = 0.f;
      for (int e = 0; e < a.E; ++e) {
        bool taken = false;
        for (int q = 0; q < r; ++q) taken |= (chosen[q] == e);
        if (taken) continue;
        const float v = l[e];
        if (best < 0 || v > bv) { best = e; bv = v; }   // strict '>' keeps the lower index on ties
      }
      chosen[r] = best;
      val[r] = bv;
    }
    float z[kMaxTopK], s = 0.f;
    for (int r = 0; r < a.k; ++r) { z[r] = expf(val[r] - val[0]); s += z[r]; }
    for (int r = 0; r < a.k; ++r) {
      a.idx[t * a.k + r] = chosen[r];
      a.w[t * a.k + r] = __half2float(__float2half_rn(z[r] / s));
    }
  }
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) { counts[e] = 0; running[e] = 0; }
  __syncthreads();
  if (a.perm == nullptr) return;
  for (int p = threadIdx.x; p < P; p += blockDim.x) atomicAdd(&counts[a.idx[p]], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0, nu = 0;
    for (int e = 0; e < a.E; ++e) {
      offs[e] = acc;
      acc += counts[e];
      if (counts[e] > 0 && a.union_list != nullptr) a.union_list[nu++] = e;
    }
    offs[a.E] = acc;
    if (a.n_union != nullptr) *a.n_union = nu;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= a.E; e += blockDim.x) a.offsets[e] = offs[e];
  // Stable placement: warp 0 walks the pairs in order, 32 at a time; equal
  // experts inside a chunk are ranked by lane (match_any + popc).
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int base = 0; base < P; base += 32) {
      const int p = base + lane;
      const bool act = p < P;
      const unsigned active = __ballot_sync(0xffffffffu, act);
      if (act) {
        const int e = a.idx[p];
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

}  // namespace

cudaError_t launch_router_logits(const RouterArgs& a, cudaStream_t s) {
  const int rows = a.E + (a.w_sg != nullptr ? 1 : 0);
  const dim3 grid(a.M, (rows + kRouterWarps - 1) / kRouterWarps);
  k_router_logits<<<grid, kRouterWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)(3 * a.E + 1) * sizeof(int);
  const int threads = a.M >= 1024 ? 1024 : ((a.M + 31) / 32) * 32 < 128 ? 128 : ((a.M + 31) / 32) * 32;
  k_route<<<1, threads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moeffn
