// Launch interface of the expert-parallel kernels (ep.cu): the routed MoE
// layer split at its two exchange points, so that the experts can live on
// other GPUs than the tokens that select them.
#pragma once
#include "common.cuh"

namespace moeffn {

// rows[s][:] = x[perm[s] / k][:] and experts[s] = idx[perm[s]] for the P = M*k
// pair slots (pairs in expert order, hence grouped by the rank owning the expert).
struct DispatchArgs {
  const uint16_t* x;   // [M][H] bf16
  const int* idx;      // [M*k] top-k experts, pair p = t*k + r
  const int* perm;     // [M*k] pair of slot s
  int P, k, H;
  uint16_t* rows;      // [P][H]
  int* experts;        // [P]
};

// Stable counting sort of R rows by local expert e = row_expert[i] - base
// (rows with e outside [0, E) are left out): offsets [E+1], perm[slot] = row
// (slots past offsets[E] hold row 0), inv[row] = slot or -1, union_list /
// n_union = experts with rows, ascending.
// One CTA; E <= kMaxExperts.
struct PlaceArgs {
  const int* row_expert;
  int R, base, E;
  int* offsets;
  int* perm;
  int* inv;
  int* union_list;
  int* n_union;
};

// out[i][:] = sum over splits s (in order, from 0) of part[s][inv[i]][:], or
// zeros where inv[i] < 0; H % 4 == 0.
struct RowsFromSlotsArgs {
  const float* part;   // [splits][slots][H]
  int splits, slots, H, R;
  const int* inv;      // [R]
  float* out;          // [R][H]
};

// inv[perm[s]] = s for s < P.
struct InvertArgs {
  const int* perm;
  int P;
  int* inv;
};

cudaError_t launch_dispatch_rows(const DispatchArgs& a, cudaStream_t s);
cudaError_t launch_place_rows(const PlaceArgs& a, cudaStream_t s);
cudaError_t launch_rows_from_slots(const RowsFromSlotsArgs& a, cudaStream_t s);
cudaError_t launch_invert_perm(const InvertArgs& a, cudaStream_t s);

}  // namespace moeffn
