// Expert-parallel pieces of the routed MoE layer: the batched pass of
// turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs
// (encode_qwen_layer_moe_batched: pair routes grouped by expert, phase 1 and
// phase 2 over the expert union, the seeded rank-ordered sum) split where
// pairs leave for the GPU that holds their expert and where the expert
// outputs come back:
//
//  * dispatch : the token row of every pair, in expert order (so grouped by
//               the rank that owns the expert), with the pair's expert;
//  * place    : on the expert's rank, the rows that arrived (from any rank,
//               in arrival order) grouped by local expert, stably;
//  * rows from slots : the grouped down projection's K-split partials summed
//               in split order and put back in arrival order (what goes back);
//  * invert   : the pair -> slot map the seeded tail reads the returned rows by.
#include <algorithm>

#include "ep.cuh"
#include "launch.cuh"
#include "route.cuh"

namespace moeffn {

namespace {

constexpr int kPlaceThreads = 1024;
constexpr int kGridCap = 148 * 8;   // grid-stride kernels: 8 CTAs per SM of a B200

__global__ void __launch_bounds__(128) k_dispatch_rows(const DispatchArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int s = blockIdx.x;
  const int p = a.perm[s];
  if (threadIdx.x == 0) a.experts[s] = a.idx[p];
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)(p / a.k) * a.H);
  uint4* dst = reinterpret_cast<uint4*>(a.rows + (size_t)s * a.H);
  for (int i = threadIdx.x; i < a.H / 8; i += blockDim.x) dst[i] = src[i];
}

// Counts per expert, offsets and union (thread 0, E <= 1024), then the rows
// placed chunk by chunk of 1024, warp by warp in row order: a warp's rows of
// one expert take consecutive slots in lane order (match_any), so the sort
// is stable. Every slot of perm is written (slots past the placed rows with
// row 0), so a consumer that reads all R slots stays inside the rows.
__global__ void __launch_bounds__(kPlaceThreads) k_place_rows(const PlaceArgs a) {
  extern __shared__ int sm[];
  int* cnt = sm;          // [E]
  int* run = sm + a.E;    // [E] next free slot of each expert
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < a.E; e += kPlaceThreads) cnt[e] = 0;
  __syncthreads();
  for (int i = tid; i < a.R; i += kPlaceThreads) {
    const int e = a.row_expert[i] - a.base;
    if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  __shared__ int placed;
  if (tid == 0) {
    int acc = 0, nu = 0;
    for (int e = 0; e < a.E; ++e) {
      a.offsets[e] = acc;
      run[e] = acc;
      if (cnt[e] > 0) a.union_list[nu++] = e;
      acc += cnt[e];
    }
    a.offsets[a.E] = acc;
    *a.n_union = nu;
    placed = acc;
  }
  __syncthreads();
  // Slots past the placed rows (rows of other ranks' experts were left out)
  // belong to no expert, but the token-row gather reads every slot: point
  // them at row 0.
  for (int s = placed + tid; s < a.R; s += kPlaceThreads) a.perm[s] = 0;
  for (int c0 = 0; c0 < a.R; c0 += kPlaceThreads) {
    const int i = c0 + tid;
    int e = -1;
    if (i < a.R) {
      e = a.row_expert[i] - a.base;
      if (e < 0 || e >= a.E) e = -1;
    }
    for (int wv = 0; wv < kPlaceThreads / 32; ++wv) {
      if (warp == wv) {
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int before = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0) {
          const int slot = run[e] + before;
          a.perm[slot] = i;
          a.inv[i] = slot;
        } else if (i < a.R) {
          a.inv[i] = -1;
        }
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) run[e] += __popc(peers);
      }
      __syncthreads();
    }
  }
}

__global__ void k_rows_from_slots(const RowsFromSlotsArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t total4 = (size_t)a.R * a.H / 4, sstride = (size_t)a.slots * a.H;
  for (size_t i4 = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i4 < total4; i4 += (size_t)gridDim.x * blockDim.x) {
    const size_t i = 4 * i4;
    const int r = (int)(i / a.H), n = (int)(i - (size_t)r * a.H);
    const int slot = a.inv[r];
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (slot >= 0) {
      for (int sp = 0; sp < a.splits; ++sp) {   // fixed split order
        const float4 p = *reinterpret_cast<const float4*>(a.part + sp * sstride + (size_t)slot * a.H + n);
        v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
      }
    }
    *reinterpret_cast<float4*>(a.out + i) = v;
  }
}

__global__ void k_invert_perm(const InvertArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < a.P; s += gridDim.x * blockDim.x) a.inv[a.perm[s]] = s;
}

}  // namespace

cudaError_t launch_dispatch_rows(const DispatchArgs& a, cudaStream_t s) {
  if (a.P <= 0) return cudaSuccess;
  return launch_pdl(k_dispatch_rows, dim3(a.P), dim3(128), 0, s, a);
}

cudaError_t launch_place_rows(const PlaceArgs& a, cudaStream_t s) {
  if (a.E < 1 || a.E > kMaxExperts) return cudaErrorInvalidValue;
  return launch_pdl(k_place_rows, dim3(1), dim3(kPlaceThreads), (size_t)2 * a.E * sizeof(int), s, a);
}

cudaError_t launch_rows_from_slots(const RowsFromSlotsArgs& a, cudaStream_t s) {
  const size_t total4 = (size_t)a.R * a.H / 4;
  if (total4 == 0) return cudaSuccess;
  const int blocks = (int)std::min<size_t>((total4 + 255) / 256, (size_t)kGridCap);
  return launch_pdl(k_rows_from_slots, dim3(blocks), dim3(256), 0, s, a);
}

cudaError_t launch_invert_perm(const InvertArgs& a, cudaStream_t s) {
  if (a.P <= 0) return cudaSuccess;
  return launch_pdl(k_invert_perm, dim3((a.P + 255) / 256), dim3(256), 0, s, a);
}

}  // namespace moeffn
