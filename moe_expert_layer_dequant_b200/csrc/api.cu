// C ABI of libmoeffn.so: argument validation, workspace carving and the
// launch sequence of each layer kind. See include/moeffn.h for the contract.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>
#include <vector>

#include "../../include/moeffn.h"
#include "common.cuh"
#include "ep.cuh"
#include "gemm_tc.cuh"
#include "gemv_tma.cuh"
#include "tmap.cuh"
#include "prof.cuh"
#include "route.cuh"
#include "tail.cuh"

using namespace moeffn;

namespace {

thread_local std::string g_last_error;

// One-shot failure injection for the next dense gate/up GEMV launch
// (moeffn_test_inject_gemv_fault; failure-detection tests only).
struct GemvInjection {
  int kind = 0;                      // 0 none, 1 producer stops, 2 ring depth
  int value = 0;
  unsigned long long wait_ns = 0;
};
GemvInjection g_inject;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(MOEFFN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define MOEFFN_CHECK_CUDA(expr, where)              \
  do {                                              \
    cudaError_t e_ = (expr);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

constexpr int kSMs = 148;
constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

QW to_qw(const moeffn_qweight& w) {
  return QW{static_cast<const uint8_t*>(w.q), static_cast<const __half*>(w.scale),
            static_cast<const __half*>(w.min)};
}

int check_qweight(const moeffn_qweight& w, const char* name, int rows, int cols) {
  if (w.format != MOEFFN_Q_INT8_ROW && w.format != MOEFFN_Q_INT4_AFFINE_G32 && w.format != MOEFFN_Q_Q4_K)
    return fail(MOEFFN_ERR_UNSUPPORTED, "%s: format %d is not INT8_ROW, INT4_AFFINE_G32 or Q4_K", name, w.format);
  if (w.rows != rows || w.cols != cols)
    return fail(MOEFFN_ERR_INVALID, "%s: shape [%d][%d], expected [%d][%d]", name, w.rows, w.cols, rows, cols);
  if (w.format == MOEFFN_Q_Q4_K) {   // scales and mins live in the blocks
    if (w.q == nullptr) return fail(MOEFFN_ERR_INVALID, "%s: null q", name);
    if (!aligned16(w.q)) return fail(MOEFFN_ERR_INVALID, "%s: q is not 16-byte aligned", name);
    if (cols % 256 != 0) return fail(MOEFFN_ERR_INVALID, "%s: Q4_K needs cols %% 256 == 0 (cols=%d)", name, cols);
    return MOEFFN_OK;
  }
  if (w.q == nullptr || w.scale == nullptr)
    return fail(MOEFFN_ERR_INVALID, "%s: null q or scale", name);
  if (!aligned16(w.q)) return fail(MOEFFN_ERR_INVALID, "%s: q is not 16-byte aligned", name);
  if ((reinterpret_cast<uintptr_t>(w.scale) & 1u) != 0) return fail(MOEFFN_ERR_INVALID, "%s: scale misaligned", name);
  if (w.format == MOEFFN_Q_INT4_AFFINE_G32) {
    if (cols % 32 != 0) return fail(MOEFFN_ERR_INVALID, "%s: INT4-affine needs cols %% 32 == 0 (cols=%d)", name, cols);
    if (w.min == nullptr) return fail(MOEFFN_ERR_INVALID, "%s: INT4-affine needs a min array", name);
    if (!aligned16(w.scale) || !aligned16(w.min))
      return fail(MOEFFN_ERR_INVALID, "%s: INT4-affine scale and min must be 16-byte aligned", name);
  } else if (cols % 16 != 0) {
    return fail(MOEFFN_ERR_INVALID, "%s: INT8 needs cols %% 16 == 0 (cols=%d)", name, cols);
  }
  return MOEFFN_OK;
}

int check_ffn(const moeffn_ffn& f, const char* name, int H, int I) {
  std::string n = name;
  int rc;
  if ((rc = check_qweight(f.gate, (n + ".gate").c_str(), I, H)) != MOEFFN_OK) return rc;
  if ((rc = check_qweight(f.up, (n + ".up").c_str(), I, H)) != MOEFFN_OK) return rc;
  if ((rc = check_qweight(f.down, (n + ".down").c_str(), H, I)) != MOEFFN_OK) return rc;
  // Block types are resolved per tensor; gate and up run in one fused kernel
  // and so share theirs, while down may differ (a mixed file).
  if (f.gate.format != f.up.format)
    return fail(MOEFFN_ERR_UNSUPPORTED, "%s: gate and up formats differ", name);
  return MOEFFN_OK;
}

// ---- launch geometry -------------------------------------------------------



// K split of a down projection: slices of at most 4096 (INT4), 3584 (Q4_K:
// 14 blocks of 18 eight-byte elements) or 2048 (INT8) elements, a multiple of
// 256 (16-byte aligned scale rows and TMA boxes of at most 256 eight-byte
// elements); every split starts below K. An INT4 matrix with K % 256 != 0
// is not split: its scale rows (K / 16 bytes apart) could not be boxed, and
// whole rows go through 1-D bulk copies.
int down_slice(int K, int fmt) {
  if (fmt == MOEFFN_Q_INT4_AFFINE_G32 && K % 256 != 0) return K;
  const int lim = fmt == MOEFFN_Q_INT8_ROW ? 2048 : fmt == MOEFFN_Q_Q4_K ? 3584 : 4096;
  const int s = (K + lim - 1) / lim;
  return ((K + s - 1) / s + 255) / 256 * 256;
}
int down_splits(int K, int fmt) {
  const int ks = down_slice(K, fmt);
  return (K + ks - 1) / ks;
}
// Partial-sum buffers are sized for the format with more splits.
int down_splits_any(int K) {
  return std::max(std::max(down_splits(K, MOEFFN_Q_INT8_ROW), down_splits(K, MOEFFN_Q_INT4_AFFINE_G32)),
                  down_splits(K, MOEFFN_Q_Q4_K));
}

// ---- TMA-fed GEMV eligibility and geometry ---------------------------------

constexpr size_t kTmaSmemBudget = 200 * 1024;
constexpr size_t kTmaXBudget = 72 * 1024;


struct TmaGeom {
  int tokens, stages, mt;
  bool ok;
};

TmaGeom tma_geom(int fmt, int nm, int klen, int want_tokens) {
  TmaGeom g{};
  g.mt = want_tokens <= 1 ? 1 : 2;
  const size_t per_tok = tma_gemv_smem(fmt, nm, klen, 1, 1, 0) - tma_gemv_smem(fmt, nm, klen, 0, 1, 0);
  int t = (int)std::max<size_t>(1, kTmaXBudget / std::max<size_t>(per_tok, 1));
  g.tokens = std::max(1, std::min(want_tokens, t));
  const size_t base = tma_gemv_smem(fmt, nm, klen, g.tokens, g.mt, 0);
  const size_t st = tma_gemv_stage_bytes(fmt, nm, klen);
  int stages = base + 2 * st <= kTmaSmemBudget ? (int)std::min<size_t>(8, (kTmaSmemBudget - base) / st) : 0;
  // Each ring slot must belong to one consumer group (see gemv_tma.cu).
  const int groups = kTmaGroups;
  stages -= stages % groups;
  g.stages = stages;
  g.ok = stages >= groups && stages >= 2;
  return g;
}

// Whether a dense FFN's weight stages fit the bulk-copy GEMV's ring (one
// token row staged; more rows are staged in blocks that fit).
bool gemv_fits(const moeffn_ffn& f, int H, int I) {
  const int fmt = f.gate.format, dfmt = f.down.format;
  return tma_geom(fmt, 2, H, 1).ok && tma_geom(dfmt, 2, down_slice(I, dfmt), 1).ok;   // down: row pairs
}

// ---- tensor-core GEMM eligibility and geometry ------------------------------

constexpr int kTcMinTokens = 6;      // dense: token rows from which the GEMM replaces the GEMV
constexpr int kTcMinMoeTokens = 8;   // MoE layer: token rows from which the grouped GEMMs are used

// The GEMM's weight stages cover 256 (INT4) or 128 (INT8) K elements, loaded
// by TMA from 16-byte aligned rows.
bool tc_ok(const moeffn_qweight& w) {
  if (!aligned16(w.q)) return false;
  if (w.format == MOEFFN_Q_INT4_AFFINE_G32) return w.cols % 256 == 0 && aligned16(w.scale) && aligned16(w.min);
  if (w.format == MOEFFN_Q_Q4_K) return w.cols % 256 == 0;
  return w.format == MOEFFN_Q_INT8_ROW && w.cols % 128 == 0 && aligned16(w.scale);
}
bool tc_ok(const moeffn_ffn& f) { return tc_ok(f.gate) && tc_ok(f.up) && tc_ok(f.down); }

// K split of a down-projection GEMM: about `want` splits, at most `max_splits`,
// slices a multiple of the weight stage K.
int tc_down_slice(int K, int fmt, int want, int max_splits) {
  const int kt = tc_k_tile(fmt);
  const int s = std::max(1, std::min(want, max_splits));
  int ks = ((K + s - 1) / s + kt - 1) / kt * kt;
  while ((K + ks - 1) / ks > max_splits) ks += kt;
  return ks;
}

// ---- workspace layout ------------------------------------------------------

struct Carve {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

struct DenseWS {
  uint16_t* acts;
  float* d;
  int* cnt;   // [kSMs] arrival counters of the down projection's K splits
  uint16_t* m;   // [M][H] the normed input, when the layer applies its input norm
};

DenseWS carve_dense(Carve& c, int M, int H, int I) {
  DenseWS w;
  w.acts = c.take<uint16_t>((size_t)M * I);
  w.d = c.take<float>((size_t)down_splits_any(I) * M * H);
  w.cnt = c.take<int>(kSMs);
  w.m = c.take<uint16_t>((size_t)M * H);
  return w;
}

struct MoeWS {
  float* logits;
  float* gate_logit;
  int* idx;
  float* w;
  int* perm;
  int* inv;
  int* offsets;
  int* union_list;
  int* n_union;
  uint16_t* acts;
  uint16_t* acts_s;
  float* d;
  float* d_s;
  uint16_t* xg;      // token rows in pair-slot order (grouped GEMM operand)
  uint16_t* m;       // [M][H] the normed input, when the layer applies its input norm
  int* route_cnt;    // [1] arrival counter of the top-k CTAs (zeroed by the router kernel)
};

// Down-projection K split shared by the routed and the shared expert jobs.
struct MoeSplit {
  int ks_len, routed, shared;
};

MoeSplit moe_split(int Ie, int Is) {
  MoeSplit s;
  s.ks_len = down_slice(std::max(Ie, Is), MOEFFN_Q_INT4_AFFINE_G32);
  s.routed = (Ie + s.ks_len - 1) / s.ks_len;
  s.shared = Is > 0 ? (Is + s.ks_len - 1) / s.ks_len : 0;
  return s;
}

MoeWS carve_moe(Carve& c, int M, int H, int Ie, int Is, int E, int k) {
  MoeWS w;
  const MoeSplit sp = moe_split(Ie, Is);
  const size_t P = (size_t)M * k;
  w.logits = c.take<float>((size_t)M * E);
  w.gate_logit = c.take<float>(M);
  w.idx = c.take<int>(P);
  w.w = c.take<float>(P);
  w.perm = c.take<int>(P);
  w.inv = c.take<int>(P);
  w.offsets = c.take<int>(E + 1);
  w.union_list = c.take<int>(E);
  w.n_union = c.take<int>(1);
  w.acts = c.take<uint16_t>(P * Ie);
  w.acts_s = c.take<uint16_t>((size_t)M * std::max(Is, 0));
  w.d = c.take<float>((size_t)sp.routed * P * H);
  w.d_s = c.take<float>((size_t)sp.shared * M * H);
  w.xg = c.take<uint16_t>(P * H);
  w.m = c.take<uint16_t>((size_t)M * H);
  w.route_cnt = c.take<int>(1);
  return w;
}

struct RouterWS {
  int* counter;      // [1] arrival counter of the top-k CTAs
  float* logits;
  int* perm;
  int* offsets;
};

RouterWS carve_router(Carve& c, int M, int E, int k) {
  RouterWS w;
  w.counter = c.take<int>(1);
  w.logits = c.take<float>((size_t)M * E);
  w.perm = c.take<int>((size_t)M * k);
  w.offsets = c.take<int>(E + 1);
  return w;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return MOEFFN_OK;
  if (ws == nullptr) return fail(MOEFFN_ERR_WORKSPACE, "workspace is null (%zu bytes needed)", need);
  if (reinterpret_cast<uintptr_t>(ws) % kAlign != 0) return fail(MOEFFN_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (ws_bytes < need) return fail(MOEFFN_ERR_WORKSPACE, "workspace %zu bytes, %zu needed", ws_bytes, need);
  return MOEFFN_OK;
}

// ---- shared FFN launch (dense mode) ---------------------------------------

// The layer's input m = rms_norm(x, norm_w) into w.m (one launch).
int launch_prenorm(const uint16_t* x, const uint16_t* norm_w, float eps, int M, int H, const DenseWS& w,
                   cudaStream_t s) {
  PrenormArgs pa{x, norm_w, eps, M, H, w.m};
  ProfScope ps("prenorm_rows", s);
  MOEFFN_CHECK_CUDA(launch_prenorm_rows(pa, s), "input norm launch");
  return MOEFFN_OK;
}

// Gate/up + activation and the down projection (fp32 K-split partials in
// w.d); returns the number of splits written through *splits_out. With `res`
// given, a path that can also applies the residual tail (*tail_done = true).
// With `norm_w`, x is the un-normed residual and the layer's input is
// m = rms_norm(x, norm_w): folded into the GEMV's activation staging, or
// written to w.m by a launch of its own before the GEMMs.
int run_dense_ffn(const moeffn_ffn& f, const uint16_t* x, int M, int H, int I, int act, const DenseWS& w,
                  cudaStream_t s, int* splits_out, uint16_t* res, bool* tail_done, const uint16_t* norm_w = nullptr,
                  float eps = 0.f) {
  *tail_done = false;
  const int fmt = f.gate.format;     // gate and up (one fused kernel)
  const int dfmt = f.down.format;    // down: its own block type
  int rc;
  if (M >= kTcMinTokens && tc_ok(f) && aligned16(x)) {
    if (norm_w != nullptr) {
      if ((rc = launch_prenorm(x, norm_w, eps, M, H, w, s)) != MOEFFN_OK) return rc;
      x = w.m;
    }
    const int ntile = tc_ntile_for(M), tt = (M + ntile - 1) / ntile;
    TcGemmArgs g{};
    g.fmt = fmt;
    g.act = act;
    g.mode = TC_GATEUP;
    g.ntile = ntile;
    g.N = I;
    g.K = H;
    g.M = M;
    g.slots = M;
    g.out_act = w.acts;
    g.ks_len = H;
    g.token_tiles = tt;
    g.rscale0 = static_cast<const __half*>(f.gate.scale);
    g.rscale1 = static_cast<const __half*>(f.up.scale);
    MOEFFN_CHECK_CUDA(encode_tc_x_map(&g.xmap, x, M, H, ntile), "tensor map encode");
    MOEFFN_CHECK_CUDA(encode_tc_weight_maps(&g.w0, fmt, to_qw(f.gate), I, H), "tensor map encode");
    MOEFFN_CHECK_CUDA(encode_tc_weight_maps(&g.w1, fmt, to_qw(f.up), I, H), "tensor map encode");
    {
      ProfScope ps("gateup_gemm_tc", s);
      MOEFFN_CHECK_CUDA(launch_tc_gemm(g, (I + kTcGateUpFeat - 1) / kTcGateUpFeat, 1, 1, s), "gate/up GEMM launch");
    }
    TcGemmArgs d{};
    d.fmt = dfmt;
    d.mode = TC_DOWN;
    d.ntile = ntile;
    d.N = H;
    d.K = I;
    d.M = M;
    d.slots = M;
    d.out_d = w.d;
    d.token_tiles = tt;
    d.rscale0 = static_cast<const __half*>(f.down.scale);
    const int row_tiles = (H + kTcDownRows - 1) / kTcDownRows;
    const int want = (kSMs + row_tiles * tt - 1) / (row_tiles * tt);
    d.ks_len = tc_down_slice(I, dfmt, want, down_splits_any(I));
    const int splits = (I + d.ks_len - 1) / d.ks_len;
    MOEFFN_CHECK_CUDA(encode_tc_x_map(&d.xmap, w.acts, M, I, ntile), "tensor map encode");
    MOEFFN_CHECK_CUDA(encode_tc_weight_maps(&d.w0, dfmt, to_qw(f.down), H, I), "tensor map encode");
    {
      ProfScope ps("down_gemm_tc", s);
      MOEFFN_CHECK_CUDA(launch_tc_gemm(d, row_tiles, splits, 1, s), "down GEMM launch");
    }
    *splits_out = splits;
    return MOEFFN_OK;
  }
  const int ks = down_slice(I, dfmt), splits = down_splits(I, dfmt);
  *splits_out = splits;
  const TmaGeom gu = tma_geom(fmt, 2, H, M);
  const TmaGeom dn = tma_geom(dfmt, 2, ks, M);   // row pairs: the two-matrix stage
  if (!gu.ok || !dn.ok)
    return fail(MOEFFN_ERR_UNSUPPORTED, "hidden size %d / intermediate size %d: the bulk-copy GEMV's stages do not fit", H, I);
  {
    TmaGemvArgs g{};
    g.fmt = fmt;
    g.act = act;
    g.a0 = to_qw(f.gate);
    g.a1 = to_qw(f.up);
    g.N = I;
    g.K = H;
    g.x = x;
    g.ld_x = H;
    g.M = M;
    g.topk = 1;
    g.routed_jobs = 1;
    g.slots = M;
    g.out_act = w.acts;
    g.ks_len = H;
    g.ctas_per_job = kSMs;
    g.stage_tokens = gu.tokens;
    g.stages = gu.stages;
    if (res != nullptr) {
      g.zero_cnt = w.cnt;
      g.zero_n = kSMs;
    }
    if (norm_w != nullptr) {
      if (gu.tokens <= kGemvNormTokens) {   // folded into the staging of the token rows
        g.norm_w = norm_w;
        g.eps = eps;
      } else {
        if ((rc = launch_prenorm(x, norm_w, eps, M, H, w, s)) != MOEFFN_OK) return rc;
        g.x = w.m;
      }
    }
    if (g_inject.kind != 0) {          // failure-detection tests only
      if (g_inject.kind == 1) g.inject_stop = g_inject.value + 1;
      if (g_inject.kind == 2) g.stages = g_inject.value;
      g.wait_ns = g_inject.wait_ns;
      g_inject = GemvInjection{};
    }
    {
      ProfScope ps("gateup_gemv_tma", s);
      MOEFFN_CHECK_CUDA(launch_tma_gemv(g, 2, gu.mt, 1, 1, s), "gate/up launch");
    }
    TmaGemvArgs d{};
    d.fmt = dfmt;
    d.a0 = to_qw(f.down);
    d.N = H;
    d.K = I;
    d.x = w.acts;
    d.ld_x = I;
    d.M = M;
    d.topk = 1;
    d.routed_jobs = 1;
    d.slots = M;
    d.out_d = w.d;
    d.ks_len = ks;
    d.use_maps = splits > 1;
    if (d.use_maps) MOEFFN_CHECK_CUDA(encode_qw_maps(&d.dmap, dfmt, to_qw(f.down), H, I, ks), "tensor map encode");
    d.ctas_per_job = std::max(1, kSMs / splits);
    d.stage_tokens = dn.tokens;
    d.stages = dn.stages;
    if (res != nullptr) {
      d.tile_cnt = w.cnt;
      d.res = res;
    }
    {
      ProfScope ps("down_gemv_tma", s);
      MOEFFN_CHECK_CUDA(launch_tma_gemv(d, 1, dn.mt, splits, 1, s), "down launch");
    }
    *tail_done = res != nullptr;
    return MOEFFN_OK;
  }

}

}  // namespace

// ============================================================================
// Plan
// ============================================================================

struct moeffn_moe_plan {
  int E, k, act, H, Ie, Is;
  int router_fmt;
  const void* router;
  const uint16_t* w_sg;
  moeffn_ffn shared;
  bool has_shared;
  const float* expert_scale = nullptr;         // per-expert routing scale (null: ones)
  const uint16_t* shared_post_norm = nullptr;  // Gemma form: the shared branch's post-FFN norm weight
  float shared_post_norm_eps = 0.f;
  QW* d_gate = nullptr;   // device tables [E]
  QW* d_up = nullptr;
  QW* d_down = nullptr;
  QWMaps* d_maps = nullptr;    // [E] tensor maps of the expert down matrices (K split)
  QWMaps* d_maps_s = nullptr;  // [1] shared expert down (K split)
  bool tc = false;             // tensor-core GEMM maps built
  TcMaps* d_tc_gate = nullptr; // [E]
  TcMaps* d_tc_up = nullptr;   // [E]
  TcMaps* d_tc_down = nullptr; // [E]
  TcMaps tc_sg{}, tc_su{}, tc_sd{};   // shared expert
};

extern "C" {

const char* moeffn_last_error(void) { return g_last_error.c_str(); }

int moeffn_test_inject_gemv_fault(int kind, int value, unsigned int wait_us) {
  g_last_error.clear();
  if (kind == 0) {
    g_inject = GemvInjection{};
    return MOEFFN_OK;
  }
  if ((kind != 1 && kind != 2) || value < 0 || (kind == 2 && (value < 1 || value > 8)) || wait_us == 0 ||
      wait_us > 1000000u)
    return fail(MOEFFN_ERR_INVALID, "moeffn_test_inject_gemv_fault: kind %d value %d wait %u us", kind, value, wait_us);
  g_inject.kind = kind;
  g_inject.value = value;
  g_inject.wait_ns = 1000ull * wait_us;
  return MOEFFN_OK;
}

unsigned int moeffn_device_faults(int clear) {
  // Blocking read of the kernels' fault words (bounded waits that ran out).
  return tma_gemv_fault_flags(clear != 0) | tc_gemm_fault_flags(clear != 0);
}

size_t moeffn_workspace_bytes(int kind, int M, int H, int I, int E, int top_k) {
  if (M < 1 || H < 1) return 0;
  Carve c{nullptr};
  switch (kind) {
    case MOEFFN_KIND_DENSE:
    case MOEFFN_KIND_SHARED:
      if (I < 1) return 0;
      carve_dense(c, M, H, I);
      return c.off;
    case MOEFFN_KIND_ROUTER:
      if (E < 1 || top_k < 1) return 0;
      carve_router(c, M, E, top_k);
      return c.off;
    case MOEFFN_KIND_MOE:
      if (I < 1 || E < 1 || top_k < 1) return 0;
      carve_moe(c, M, H, I, I, E, top_k);
      return c.off;
    default:
      return 0;
  }
}

namespace {

// ffn_dense and ffn_dense_prenorm: with norm_w, x is null and the input is
// m = rms_norm(residual, norm_w).
int dense_entry(const char* who, const moeffn_ffn* w, const uint16_t* x, const uint16_t* norm_w, float eps,
                uint16_t* residual, int M, int act, void* ws, size_t ws_bytes, moeffn_stream_t stream) {
  g_last_error.clear();
  if (w == nullptr || residual == nullptr || (x == nullptr && norm_w == nullptr))
    return fail(MOEFFN_ERR_INVALID, "%s: null pointer", who);
  if (M < 1) return fail(MOEFFN_ERR_INVALID, "%s: M=%d", who, M);
  if (act != MOEFFN_ACT_SILU && act != MOEFFN_ACT_GELU_TANH) return fail(MOEFFN_ERR_INVALID, "%s: act=%d", who, act);
  const int H = w->gate.cols, I = w->gate.rows;
  int rc = check_ffn(*w, who, H, I);
  if (rc != MOEFFN_OK) return rc;
  if (norm_w != nullptr) {
    if (!aligned16(norm_w)) return fail(MOEFFN_ERR_INVALID, "%s: norm weight not 16-byte aligned", who);
    if (!(eps >= 0.0f)) return fail(MOEFFN_ERR_INVALID, "%s: eps must be >= 0", who);
    x = residual;
  }
  if (!aligned16(x) || !aligned16(residual)) return fail(MOEFFN_ERR_INVALID, "%s: x/residual not 16-byte aligned", who);
  if (norm_w == nullptr && x == residual) return fail(MOEFFN_ERR_INVALID, "%s: x aliases residual", who);
  if (!gemv_fits(*w, H, I))
    return fail(MOEFFN_ERR_UNSUPPORTED, "%s: hidden size %d too large for the bulk-copy GEMV's stages", who, H);
  Carve c{nullptr};
  carve_dense(c, M, H, I);
  if ((rc = check_ws(ws, ws_bytes, c.off)) != MOEFFN_OK) return rc;
  Carve cw{static_cast<char*>(ws)};
  const DenseWS d = carve_dense(cw, M, H, I);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int splits = 0;
  bool tail_done = false;
  if ((rc = run_dense_ffn(*w, x, M, H, I, act, d, s, &splits, residual, &tail_done, norm_w, eps)) != MOEFFN_OK)
    return rc;
  if (tail_done) return MOEFFN_OK;
  TailArgs t{};
  t.mode = TAIL_RESIDUAL;
  t.M = M;
  t.N = H;
  t.d = d.d;
  t.splits = splits;
  t.slots = M;
  t.res = residual;
  {
    ProfScope ps("tail_residual", s);
    MOEFFN_CHECK_CUDA(launch_tail(t, s), "residual tail launch");
  }
  return MOEFFN_OK;
}

}  // namespace

int ffn_dense(const moeffn_ffn* w, const uint16_t* x, uint16_t* residual, int M, int act, void* ws,
              size_t ws_bytes, moeffn_stream_t stream) {
  if (x == nullptr) return fail(MOEFFN_ERR_INVALID, "ffn_dense: null pointer");
  return dense_entry("ffn_dense", w, x, nullptr, 0.f, residual, M, act, ws, ws_bytes, stream);
}

int ffn_dense_prenorm(const moeffn_ffn* w, const uint16_t* norm_w, float eps, uint16_t* residual, int M, int act,
                      void* ws, size_t ws_bytes, moeffn_stream_t stream) {
  if (norm_w == nullptr) return fail(MOEFFN_ERR_INVALID, "ffn_dense_prenorm: null norm weight");
  return dense_entry("ffn_dense_prenorm", w, nullptr, norm_w, eps, residual, M, act, ws, ws_bytes, stream);
}

int ffn_shared_expert(const moeffn_ffn* w, const uint16_t* x, const uint16_t* norm_w, float eps, uint16_t* h1_out,
                      int M, int act, void* ws, size_t ws_bytes, moeffn_stream_t stream) {
  g_last_error.clear();
  if (w == nullptr || x == nullptr || norm_w == nullptr || h1_out == nullptr)
    return fail(MOEFFN_ERR_INVALID, "ffn_shared_expert: null pointer");
  if (M < 1) return fail(MOEFFN_ERR_INVALID, "ffn_shared_expert: M=%d", M);
  if (act != MOEFFN_ACT_SILU && act != MOEFFN_ACT_GELU_TANH)
    return fail(MOEFFN_ERR_INVALID, "ffn_shared_expert: act=%d", act);
  if (!(eps >= 0.0f)) return fail(MOEFFN_ERR_INVALID, "ffn_shared_expert: eps must be >= 0");
  const int H = w->gate.cols, I = w->gate.rows;
  int rc = check_ffn(*w, "ffn_shared_expert", H, I);
  if (rc != MOEFFN_OK) return rc;
  if (!aligned16(x) || !aligned16(h1_out)) return fail(MOEFFN_ERR_INVALID, "ffn_shared_expert: x/h1 not 16-byte aligned");
  if (x == h1_out) return fail(MOEFFN_ERR_INVALID, "ffn_shared_expert: x aliases h1_out");
  if (!gemv_fits(*w, H, I))
    return fail(MOEFFN_ERR_UNSUPPORTED, "ffn_shared_expert: hidden size %d too large for the bulk-copy GEMV's stages", H);
  Carve c{nullptr};
  carve_dense(c, M, H, I);
  if ((rc = check_ws(ws, ws_bytes, c.off)) != MOEFFN_OK) return rc;
  Carve cw{static_cast<char*>(ws)};
  const DenseWS d = carve_dense(cw, M, H, I);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int splits = 0;
  bool tail_done = false;
  if ((rc = run_dense_ffn(*w, x, M, H, I, act, d, s, &splits, nullptr, &tail_done)) != MOEFFN_OK) return rc;
  TailArgs t{};
  t.mode = TAIL_RMSNORM;
  t.M = M;
  t.N = H;
  t.d = d.d;
  t.splits = splits;
  t.slots = M;
  t.h1 = h1_out;
  t.norm_w = norm_w;
  t.eps = eps;
  {
    ProfScope ps("tail_rmsnorm", s);
    MOEFFN_CHECK_CUDA(launch_tail(t, s), "rmsnorm tail launch");
  }
  return MOEFFN_OK;
}

static int check_router(const moeffn_qweight* router, int H_expected, const char* who) {
  if (router == nullptr || router->q == nullptr) return fail(MOEFFN_ERR_INVALID, "%s: null router", who);
  if (router->format != MOEFFN_F32 && router->format != MOEFFN_BF16)
    return fail(MOEFFN_ERR_UNSUPPORTED, "%s: router format %d is not F32 or BF16", who, router->format);
  if (router->rows < 1 || router->rows > kMaxExperts)
    return fail(MOEFFN_ERR_UNSUPPORTED, "%s: %d experts (1..%d supported)", who, router->rows, kMaxExperts);
  if (H_expected >= 0 && router->cols != H_expected)
    return fail(MOEFFN_ERR_INVALID, "%s: router cols %d != hidden %d", who, router->cols, H_expected);
  if (router->cols % 8 != 0) return fail(MOEFFN_ERR_INVALID, "%s: hidden size must be a multiple of 8", who);
  if (!aligned16(router->q)) return fail(MOEFFN_ERR_INVALID, "%s: router not 16-byte aligned", who);
  return MOEFFN_OK;
}

int moe_router_topk(const moeffn_qweight* router, const uint16_t* x, int M, int top_k, float* logits_out,
                    int32_t* topk_idx, float* topk_w, int32_t* perm, int32_t* expert_offsets, void* ws,
                    size_t ws_bytes, moeffn_stream_t stream) {
  g_last_error.clear();
  int rc = check_router(router, -1, "moe_router_topk");
  if (rc != MOEFFN_OK) return rc;
  const int E = router->rows, H = router->cols;
  if (x == nullptr || topk_idx == nullptr || topk_w == nullptr) return fail(MOEFFN_ERR_INVALID, "moe_router_topk: null pointer");
  if (!aligned16(x)) return fail(MOEFFN_ERR_INVALID, "moe_router_topk: x not 16-byte aligned");
  if (M < 1) return fail(MOEFFN_ERR_INVALID, "moe_router_topk: M=%d", M);
  if (top_k < 1 || top_k > kMaxTopK || top_k > E)
    return fail(MOEFFN_ERR_UNSUPPORTED, "moe_router_topk: top_k=%d (1..%d and <= E=%d)", top_k, kMaxTopK, E);
  if (perm != nullptr && expert_offsets == nullptr)
    return fail(MOEFFN_ERR_INVALID, "moe_router_topk: perm needs expert_offsets");
  Carve c{nullptr};
  carve_router(c, M, E, top_k);
  if ((rc = check_ws(ws, ws_bytes, c.off)) != MOEFFN_OK) return rc;
  Carve cw{static_cast<char*>(ws)};
  const RouterWS w = carve_router(cw, M, E, top_k);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RouterArgs ra{};
  ra.router = router->q;
  ra.router_f32 = router->format == MOEFFN_F32;
  ra.x = x;
  ra.M = M;
  ra.H = H;
  ra.E = E;
  ra.logits = logits_out != nullptr ? logits_out : w.logits;
  ra.route_cnt = w.counter;
  {
    ProfScope ps("router_logits", s);
    MOEFFN_CHECK_CUDA(launch_router_logits(ra, s), "router launch");
  }
  RouteArgs rt{};
  rt.logits = ra.logits;
  rt.M = M;
  rt.E = E;
  rt.k = top_k;
  rt.idx = topk_idx;
  rt.w = topk_w;
  rt.perm = perm;
  rt.offsets = expert_offsets;
  rt.counter = w.counter;
  {
    ProfScope ps("route_topk", s);
    MOEFFN_CHECK_CUDA(launch_route(rt, s), "top-k launch");
  }
  return MOEFFN_OK;
}

int moe_plan_create(const moeffn_moe_desc* desc, moeffn_moe_plan** plan) {
  g_last_error.clear();
  if (desc == nullptr || plan == nullptr) return fail(MOEFFN_ERR_INVALID, "moe_plan_create: null pointer");
  *plan = nullptr;
  int rc = check_router(&desc->router, -1, "moe_plan_create");
  if (rc != MOEFFN_OK) return rc;
  const int E = desc->num_experts, k = desc->top_k, H = desc->router.cols;
  if (E != desc->router.rows) return fail(MOEFFN_ERR_INVALID, "moe_plan_create: num_experts %d != router rows %d", E, desc->router.rows);
  if (k < 1 || k > kMaxTopK || k > E) return fail(MOEFFN_ERR_UNSUPPORTED, "moe_plan_create: top_k=%d", k);
  if (desc->act != MOEFFN_ACT_SILU && desc->act != MOEFFN_ACT_GELU_TANH)
    return fail(MOEFFN_ERR_INVALID, "moe_plan_create: act=%d", desc->act);
  if (desc->experts == nullptr) return fail(MOEFFN_ERR_INVALID, "moe_plan_create: null experts");
  const int Ie = desc->experts[0].gate.rows;
  std::vector<QW> g(E), u(E), d(E);
  for (int e = 0; e < E; ++e) {
    char name[64];
    snprintf(name, sizeof(name), "expert[%d]", e);
    if ((rc = check_ffn(desc->experts[e], name, H, Ie)) != MOEFFN_OK) return rc;
    if (desc->experts[e].gate.format != MOEFFN_Q_INT4_AFFINE_G32)
      return fail(MOEFFN_ERR_UNSUPPORTED, "moe_plan_create: %s is not INT4-affine (the routed path takes INT4-affine blobs only)", name);
    g[e] = to_qw(desc->experts[e].gate);
    u[e] = to_qw(desc->experts[e].up);
    d[e] = to_qw(desc->experts[e].down);
  }
  int Is = 0;
  if (desc->shared != nullptr) {
    Is = desc->shared->gate.rows;
    if ((rc = check_ffn(*desc->shared, "shared", H, Is)) != MOEFFN_OK) return rc;
    if (desc->shared->gate.format != MOEFFN_Q_INT4_AFFINE_G32)
      return fail(MOEFFN_ERR_UNSUPPORTED, "moe_plan_create: the shared expert must be INT4-affine like the routed ones");
    if (desc->shared_post_norm != nullptr) {   // Gemma form: normed, ungated shared branch
      if (desc->shared_gate != nullptr)
        return fail(MOEFFN_ERR_INVALID, "moe_plan_create: the Gemma form (shared_post_norm) has no shared_gate");
      if (!aligned16(desc->shared_post_norm) || !(desc->shared_post_norm_eps >= 0.0f))
        return fail(MOEFFN_ERR_INVALID, "moe_plan_create: shared_post_norm not 16-byte aligned or eps < 0");
    } else if (desc->shared_gate == nullptr || desc->shared_gate->q == nullptr || desc->shared_gate->format != MOEFFN_BF16 ||
               desc->shared_gate->cols != H || desc->shared_gate->rows != 1 || !aligned16(desc->shared_gate->q)) {
      return fail(MOEFFN_ERR_INVALID, "moe_plan_create: shared expert needs a BF16 [1][H] 16-byte aligned shared_gate");
    }
  } else if (desc->shared_gate != nullptr || desc->shared_post_norm != nullptr) {
    return fail(MOEFFN_ERR_INVALID, "moe_plan_create: shared_gate / shared_post_norm without a shared expert");
  }
  if (desc->expert_scale != nullptr && (reinterpret_cast<uintptr_t>(desc->expert_scale) & 3u) != 0)
    return fail(MOEFFN_ERR_INVALID, "moe_plan_create: expert_scale not 4-byte aligned");
  if (!tma_geom(MOEFFN_Q_INT4_AFFINE_G32, 2, H, 1).ok ||
      !tma_geom(MOEFFN_Q_INT4_AFFINE_G32, 2, moe_split(Ie, Is).ks_len, 1).ok)
    return fail(MOEFFN_ERR_UNSUPPORTED, "moe_plan_create: hidden size %d too large for the bulk-copy GEMV's stages", H);
  auto* p = new moeffn_moe_plan();
  p->E = E; p->k = k; p->act = desc->act; p->H = H; p->Ie = Ie; p->Is = Is;
  p->router_fmt = desc->router.format;
  p->router = desc->router.q;
  p->has_shared = desc->shared != nullptr;
  if (p->has_shared) {
    p->shared = *desc->shared;
    p->w_sg = desc->shared_gate != nullptr ? static_cast<const uint16_t*>(desc->shared_gate->q) : nullptr;
  }
  p->expert_scale = desc->expert_scale;
  p->shared_post_norm = desc->shared_post_norm;
  p->shared_post_norm_eps = desc->shared_post_norm_eps;
  cudaError_t e1 = cudaMalloc(&p->d_gate, sizeof(QW) * E);
  cudaError_t e2 = cudaMalloc(&p->d_up, sizeof(QW) * E);
  cudaError_t e3 = cudaMalloc(&p->d_down, sizeof(QW) * E);
  if (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) {
    moe_plan_destroy(p);
    return fail(MOEFFN_ERR_CUDA, "moe_plan_create: cudaMalloc of the pointer tables failed");
  }
  cudaError_t e4 = cudaMemcpy(p->d_gate, g.data(), sizeof(QW) * E, cudaMemcpyHostToDevice);
  cudaError_t e5 = cudaMemcpy(p->d_up, u.data(), sizeof(QW) * E, cudaMemcpyHostToDevice);
  cudaError_t e6 = cudaMemcpy(p->d_down, d.data(), sizeof(QW) * E, cudaMemcpyHostToDevice);
  if (e4 != cudaSuccess || e5 != cudaSuccess || e6 != cudaSuccess) {
    moe_plan_destroy(p);
    return fail(MOEFFN_ERR_CUDA, "moe_plan_create: copy of the pointer tables failed");
  }
  // Tensor maps for the down projections split along K (bulk-copy GEMV).
  const MoeSplit sp = moe_split(Ie, Is);
  if (sp.routed > 1 || sp.shared > 1) {
    std::vector<QWMaps> maps(E);
    bool ok = true;
    for (int e = 0; e < E && ok; ++e)
      ok = encode_qw_maps(&maps[e], MOEFFN_Q_INT4_AFFINE_G32, d[e], H, Ie, sp.ks_len) == cudaSuccess;
    QWMaps ms{};
    if (ok && p->has_shared && sp.shared > 1)
      ok = encode_qw_maps(&ms, MOEFFN_Q_INT4_AFFINE_G32, to_qw(p->shared.down), H, Is, sp.ks_len) == cudaSuccess;
    if (!ok) {
      moe_plan_destroy(p);
      return fail(MOEFFN_ERR_CUDA, "moe_plan_create: tensor map encoding failed");
    }
    if (cudaMalloc(&p->d_maps, sizeof(QWMaps) * E) != cudaSuccess ||
        cudaMemcpy(p->d_maps, maps.data(), sizeof(QWMaps) * E, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMalloc(&p->d_maps_s, sizeof(QWMaps)) != cudaSuccess ||
        cudaMemcpy(p->d_maps_s, &ms, sizeof(QWMaps), cudaMemcpyHostToDevice) != cudaSuccess) {
      moe_plan_destroy(p);
      return fail(MOEFFN_ERR_CUDA, "moe_plan_create: tensor map upload failed");
    }
  }
  // Tensor maps of the grouped tensor-core GEMMs.
  bool tc = true;
  for (int e = 0; e < E && tc; ++e) tc = tc_ok(desc->experts[e]);
  if (tc && p->has_shared) tc = tc_ok(*desc->shared);
  if (tc) {
    std::vector<TcMaps> tg(E), tu(E), td(E);
    bool ok = true;
    for (int e = 0; e < E && ok; ++e) {
      ok = encode_tc_weight_maps(&tg[e], MOEFFN_Q_INT4_AFFINE_G32, g[e], Ie, H) == cudaSuccess &&
           encode_tc_weight_maps(&tu[e], MOEFFN_Q_INT4_AFFINE_G32, u[e], Ie, H) == cudaSuccess &&
           encode_tc_weight_maps(&td[e], MOEFFN_Q_INT4_AFFINE_G32, d[e], H, Ie) == cudaSuccess;
    }
    if (ok && p->has_shared) {
      ok = encode_tc_weight_maps(&p->tc_sg, MOEFFN_Q_INT4_AFFINE_G32, to_qw(p->shared.gate), Is, H) == cudaSuccess &&
           encode_tc_weight_maps(&p->tc_su, MOEFFN_Q_INT4_AFFINE_G32, to_qw(p->shared.up), Is, H) == cudaSuccess &&
           encode_tc_weight_maps(&p->tc_sd, MOEFFN_Q_INT4_AFFINE_G32, to_qw(p->shared.down), H, Is) == cudaSuccess;
    }
    const size_t bytes = sizeof(TcMaps) * E;
    if (!ok || cudaMalloc(&p->d_tc_gate, bytes) != cudaSuccess || cudaMalloc(&p->d_tc_up, bytes) != cudaSuccess ||
        cudaMalloc(&p->d_tc_down, bytes) != cudaSuccess ||
        cudaMemcpy(p->d_tc_gate, tg.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(p->d_tc_up, tu.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(p->d_tc_down, td.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
      moe_plan_destroy(p);
      return fail(MOEFFN_ERR_CUDA, "moe_plan_create: tensor-core GEMM maps failed");
    }
    p->tc = true;
  }
  *plan = p;
  return MOEFFN_OK;
}

int moe_plan_destroy(moeffn_moe_plan* plan) {
  if (plan == nullptr) return MOEFFN_OK;
  cudaFree(plan->d_gate);
  cudaFree(plan->d_up);
  cudaFree(plan->d_down);
  cudaFree(plan->d_maps);
  cudaFree(plan->d_maps_s);
  cudaFree(plan->d_tc_gate);
  cudaFree(plan->d_tc_up);
  cudaFree(plan->d_tc_down);
  delete plan;
  return MOEFFN_OK;
}

size_t moe_workspace_bytes(const moeffn_moe_plan* p, int M) {
  if (p == nullptr || M < 1) return 0;
  Carve c{nullptr};
  carve_moe(c, M, p->H, p->Ie, p->Is, p->E, p->k);
  return c.off;
}

namespace {

// Phase 1 (grouped gate/up + activation) and phase 2 (grouped down into the
// fp32 K-split partials w.d, w.d_s) over the pairs grouped in w (perm, offsets,
// union_list, n_union): pair slot i reads token row perm[i] / k of x. With
// use_shared the plan's shared expert runs as one more job over all M rows.
// The split counts of w.d and w.d_s go to *splits_r_out and *splits_s_out.
int run_moe_phases(moeffn_moe_plan* p, const uint16_t* x, int M, int k, const MoeWS& w, bool use_shared,
                   cudaStream_t s, int* splits_r_out, int* splits_s_out) {
  const int E = p->E, H = p->H, Ie = p->Ie, Is = p->Is;
  const int P = M * k;
  const int routed_jobs = std::min(E, P);
  const int jobs = routed_jobs + (use_shared ? 1 : 0);
  const int max_tok = M;  // a token selects an expert at most once
  const MoeSplit sp = moe_split(Ie, Is);
  const int splits_r = sp.routed, splits_sh = sp.shared;
  const int splits = std::max(splits_r, splits_sh);
  const TmaGeom gu = tma_geom(MOEFFN_Q_INT4_AFFINE_G32, 2, H, max_tok);
  const TmaGeom dn = tma_geom(MOEFFN_Q_INT4_AFFINE_G32, 2, sp.ks_len, max_tok);   // row pairs
  int tc_splits_r = splits_r, tc_splits_s = splits_sh;
  const bool use_tc = p->tc && M >= kTcMinMoeTokens && aligned16(x);
  if (use_tc) {
    // Token rows in pair-slot order feed phase 1's B operand.
    GatherArgs ga{x, w.perm, k, H, P, w.xg};
    {
      ProfScope ps("gather_rows", s);
      MOEFFN_CHECK_CUDA(launch_gather_rows(ga, s), "gather launch");
    }
    // One CTA should cover a whole expert's token rows, since a second token
    // tile dequantizes every weight of the expert again: the token tile is
    // sized for the mean load per expert plus the larger of a quarter of it
    // and 2.5 standard deviations of the routing spread (about sqrt(mean)); an
    // expert holds at most M rows. Keeping the tile narrow leaves TMEM for a
    // deeper A stage ring (a tile of 160 columns leaves three stages, 192 two).
    const int per_expert = std::max(1, P / std::min(E, P));
    const int spread = std::max(per_expert / 4, (int)(2.5 * std::sqrt((double)per_expert)) + 1);
    const int ntile = std::min(kTcMaxTok, (std::min(M, per_expert + spread) + 15) & ~15);
    const int tt = (M + ntile - 1) / ntile;
    TcGemmArgs g{};
    g.fmt = MOEFFN_Q_INT4_AFFINE_G32;
    g.act = p->act;
    g.mode = TC_GATEUP;
    g.ntile = ntile;
    g.N = Ie;
    g.K = H;
    g.Ns = Is;
    g.Ks = H;
    g.M = M;
    g.offsets = w.offsets;
    g.union_list = w.union_list;
    g.n_union = w.n_union;
    g.routed_jobs = routed_jobs;
    g.slots = P;
    g.tab0 = p->d_tc_gate;
    g.tab1 = p->d_tc_up;
    g.s0 = p->tc_sg;
    g.s1 = p->tc_su;
    g.out_act = w.acts;
    g.out_act_s = w.acts_s;
    g.ks_len = H;
    g.token_tiles = tt;
    MOEFFN_CHECK_CUDA(encode_tc_x_map(&g.xmap, w.xg, P, H, ntile), "tensor map encode");
    MOEFFN_CHECK_CUDA(encode_tc_x_map(&g.xmap_s, x, M, H, ntile), "tensor map encode");
    const int rt1 = (std::max(Ie, Is) + kTcGateUpFeat - 1) / kTcGateUpFeat;
    {
      ProfScope ps("phase1_gateup_gemm_tc", s);
      MOEFFN_CHECK_CUDA(launch_tc_gemm(g, rt1, 1, jobs, s), "phase-1 GEMM launch");
    }
    TcGemmArgs d{};
    d.fmt = MOEFFN_Q_INT4_AFFINE_G32;
    d.mode = TC_DOWN;
    d.ntile = ntile;
    d.N = H;
    d.K = Ie;
    d.Ns = H;
    d.Ks = Is;
    d.M = M;
    d.offsets = w.offsets;
    d.union_list = w.union_list;
    d.n_union = w.n_union;
    d.routed_jobs = routed_jobs;
    d.slots = P;
    d.tab0 = p->d_tc_down;
    d.s0 = p->tc_sd;
    d.out_d = w.d;
    d.out_d_s = w.d_s;
    d.token_tiles = tt;
    const int row_tiles = (H + kTcDownRows - 1) / kTcDownRows;
    const int active = std::max(1, std::min(E, P)) * std::max(1, (per_expert + ntile - 1) / ntile);
    const int want = (kSMs + row_tiles * active - 1) / (row_tiles * active);
    d.ks_len = tc_down_slice(Ie, MOEFFN_Q_INT4_AFFINE_G32, want, sp.routed);
    tc_splits_r = (Ie + d.ks_len - 1) / d.ks_len;
    tc_splits_s = Is > 0 ? (Is + d.ks_len - 1) / d.ks_len : 0;
    if (tc_splits_s > sp.shared) {   // keep within the workspace's partial buffers
      d.ks_len = sp.ks_len;
      tc_splits_r = splits_r;
      tc_splits_s = splits_sh;
    }
    MOEFFN_CHECK_CUDA(encode_tc_x_map(&d.xmap, w.acts, P, Ie, ntile), "tensor map encode");
    if (Is > 0) MOEFFN_CHECK_CUDA(encode_tc_x_map(&d.xmap_s, w.acts_s, M, Is, ntile), "tensor map encode");
    {
      ProfScope ps("phase2_down_gemm_tc", s);
      MOEFFN_CHECK_CUDA(launch_tc_gemm(d, row_tiles, std::max(tc_splits_r, tc_splits_s), jobs, s),
                        "phase-2 GEMM launch");
    }
  } else {
    TmaGemvArgs g{};
    g.fmt = MOEFFN_Q_INT4_AFFINE_G32;
    g.act = p->act;
    g.tab0 = p->d_gate;
    g.tab1 = p->d_up;
    if (use_shared) {
      g.s0 = to_qw(p->shared.gate);
      g.s1 = to_qw(p->shared.up);
      g.Ns = Is;
      g.Ks = H;
    }
    g.N = Ie;
    g.K = H;
    g.x = x;
    g.ld_x = H;
    g.x_s = x;
    g.M = M;
    g.topk = k;
    g.perm = w.perm;
    g.offsets = w.offsets;
    g.union_list = w.union_list;
    g.n_union = w.n_union;
    g.routed_jobs = routed_jobs;
    g.slots = P;
    g.out_act = w.acts;
    g.out_act_s = w.acts_s;
    g.ks_len = H;
    g.ctas_per_job = std::max(1, kSMs / jobs);
    g.stage_tokens = gu.tokens;
    g.stages = gu.stages;
    {
      ProfScope ps("phase1_gateup_gemv_tma", s);
      MOEFFN_CHECK_CUDA(launch_tma_gemv(g, 2, gu.mt, 1, jobs, s), "phase-1 launch");
    }
    TmaGemvArgs d{};
    d.fmt = MOEFFN_Q_INT4_AFFINE_G32;
    d.tab0 = p->d_down;
    if (use_shared) {
      d.s0 = to_qw(p->shared.down);
      d.Ns = H;
      d.Ks = Is;
    }
    d.N = H;
    d.K = Ie;
    d.x = w.acts;
    d.ld_x = Ie;
    d.x_s = w.acts_s;
    d.M = M;
    d.topk = k;
    d.offsets = w.offsets;
    d.union_list = w.union_list;
    d.n_union = w.n_union;
    d.routed_jobs = routed_jobs;
    d.slots = P;
    d.out_d = w.d;
    d.out_d_s = w.d_s;
    d.ks_len = sp.ks_len;
    d.use_maps = splits > 1;
    d.maps = p->d_maps;
    d.maps_s = p->d_maps_s;
    d.ctas_per_job = std::max(1, kSMs / (jobs * splits));
    d.stage_tokens = dn.tokens;
    d.stages = dn.stages;
    {
      ProfScope ps("phase2_down_gemv_tma", s);
      MOEFFN_CHECK_CUDA(launch_tma_gemv(d, 1, dn.mt, splits, jobs, s), "phase-2 launch");
    }
  }

  *splits_r_out = tc_splits_r;
  *splits_s_out = tc_splits_s;
  return MOEFFN_OK;
}

// moe_layer and moe_layer_prenorm: with norm_w, x is null and the input is
// m = rms_norm(residual, norm_w), formed by the router kernel.
int moe_entry(const char* who, moeffn_moe_plan* p, const uint16_t* x, const uint16_t* norm_w, float eps,
              uint16_t* residual, int M, int32_t* topk_idx_out, void* ws, size_t ws_bytes, moeffn_stream_t stream) {
  g_last_error.clear();
  if (p == nullptr || residual == nullptr || (x == nullptr && norm_w == nullptr))
    return fail(MOEFFN_ERR_INVALID, "%s: null pointer", who);
  if (M < 1) return fail(MOEFFN_ERR_INVALID, "%s: M=%d", who, M);
  if (norm_w != nullptr) {
    if (!aligned16(norm_w)) return fail(MOEFFN_ERR_INVALID, "%s: norm weight not 16-byte aligned", who);
    if (!(eps >= 0.0f)) return fail(MOEFFN_ERR_INVALID, "%s: eps must be >= 0", who);
  }
  if ((x != nullptr && !aligned16(x)) || !aligned16(residual))
    return fail(MOEFFN_ERR_INVALID, "%s: x/residual not 16-byte aligned", who);
  if (x == residual) return fail(MOEFFN_ERR_INVALID, "%s: x aliases residual", who);
  const int E = p->E, k = p->k, H = p->H, Ie = p->Ie, Is = p->Is;
  Carve c{nullptr};
  carve_moe(c, M, H, Ie, Is, E, k);
  int rc = check_ws(ws, ws_bytes, c.off);
  if (rc != MOEFFN_OK) return rc;
  Carve cw{static_cast<char*>(ws)};
  const MoeWS w = carve_moe(cw, M, H, Ie, Is, E, k);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int P = M * k;

  RouterArgs ra{};
  ra.router = p->router;
  ra.router_f32 = p->router_fmt == MOEFFN_F32;
  ra.w_sg = p->has_shared ? p->w_sg : nullptr;   // null in the Gemma form (no gate)
  ra.x = norm_w != nullptr ? residual : x;
  ra.M = M;
  ra.H = H;
  ra.E = E;
  ra.logits = w.logits;
  ra.gate_logit = w.gate_logit;
  ra.route_cnt = w.route_cnt;
  if (norm_w != nullptr) {   // the router kernel forms m for every later step
    ra.norm_w = norm_w;
    ra.eps = eps;
    ra.m_out = w.m;
    x = w.m;
  }
  {
    ProfScope ps("router_logits", s);
    MOEFFN_CHECK_CUDA(launch_router_logits(ra, s), "router launch");
  }

  RouteArgs rt{};
  rt.logits = w.logits;
  rt.M = M;
  rt.E = E;
  rt.k = k;
  rt.idx = topk_idx_out != nullptr ? topk_idx_out : w.idx;
  rt.w = w.w;
  rt.perm = w.perm;
  rt.inv = w.inv;
  rt.offsets = w.offsets;
  rt.union_list = w.union_list;
  rt.n_union = w.n_union;
  rt.scale = p->expert_scale;
  rt.counter = w.route_cnt;
  {
    ProfScope ps("route_topk", s);
    MOEFFN_CHECK_CUDA(launch_route(rt, s), "route launch");
  }

  int tc_splits_r = 0, tc_splits_s = 0;
  if ((rc = run_moe_phases(p, x, M, k, w, p->has_shared, s, &tc_splits_r, &tc_splits_s)) != MOEFFN_OK) return rc;
  TailArgs t{};
  t.mode = p->shared_post_norm != nullptr ? TAIL_MOE_GEMMA : TAIL_MOE;
  t.norm_w = p->shared_post_norm;
  t.eps = p->shared_post_norm_eps;
  t.M = M;
  t.N = H;
  t.d = w.d;
  t.splits = tc_splits_r;
  t.slots = P;
  t.d_s = p->has_shared ? w.d_s : nullptr;
  t.splits_s = tc_splits_s;
  t.gate_logit = w.gate_logit;
  t.w = w.w;
  t.inv = w.inv;
  t.k = k;
  t.res = residual;
  {
    ProfScope ps("tail_moe", s);
    MOEFFN_CHECK_CUDA(launch_tail(t, s), "moe tail launch");
  }
  return MOEFFN_OK;
}

}  // namespace

int moe_layer(moeffn_moe_plan* p, const uint16_t* x, uint16_t* residual, int M, int32_t* topk_idx_out, void* ws,
              size_t ws_bytes, moeffn_stream_t stream) {
  if (x == nullptr) return fail(MOEFFN_ERR_INVALID, "moe_layer: null pointer");
  return moe_entry("moe_layer", p, x, nullptr, 0.f, residual, M, topk_idx_out, ws, ws_bytes, stream);
}

int moe_layer_prenorm(moeffn_moe_plan* p, const uint16_t* norm_w, float eps, uint16_t* residual, int M,
                      int32_t* topk_idx_out, void* ws, size_t ws_bytes, moeffn_stream_t stream) {
  if (norm_w == nullptr) return fail(MOEFFN_ERR_INVALID, "moe_layer_prenorm: null norm weight");
  return moe_entry("moe_layer_prenorm", p, nullptr, norm_w, eps, residual, M, topk_idx_out, ws, ws_bytes, stream);
}

// ---- expert-parallel pieces ------------------------------------------------

int moe_dispatch_rows(const uint16_t* x, const int32_t* topk_idx, const int32_t* perm, int M, int top_k, int H,
                      uint16_t* rows_out, int32_t* expert_out, moeffn_stream_t stream) {
  g_last_error.clear();
  if (x == nullptr || topk_idx == nullptr || perm == nullptr || rows_out == nullptr || expert_out == nullptr)
    return fail(MOEFFN_ERR_INVALID, "moe_dispatch_rows: null pointer");
  if (M < 1 || top_k < 1 || top_k > kMaxTopK || H < 8 || H % 8 != 0)
    return fail(MOEFFN_ERR_INVALID, "moe_dispatch_rows: M=%d top_k=%d H=%d (H a positive multiple of 8)", M, top_k, H);
  if (!aligned16(x) || !aligned16(rows_out)) return fail(MOEFFN_ERR_INVALID, "moe_dispatch_rows: x/rows_out not 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DispatchArgs a{x, topk_idx, perm, M * top_k, top_k, H, rows_out, expert_out};
  ProfScope ps("dispatch_rows", s);
  MOEFFN_CHECK_CUDA(launch_dispatch_rows(a, s), "dispatch launch");
  return MOEFFN_OK;
}

size_t moe_experts_workspace_bytes(const moeffn_moe_plan* p, int R) {
  if (p == nullptr || R < 1) return 0;
  Carve c{nullptr};
  carve_moe(c, R, p->H, p->Ie, p->Is, p->E, 1);
  return c.off;
}

int moe_experts_grouped(moeffn_moe_plan* p, const uint16_t* rows, int R, const int32_t* row_expert,
                        int expert_base, float* d_out, void* ws, size_t ws_bytes, moeffn_stream_t stream) {
  g_last_error.clear();
  if (p == nullptr) return fail(MOEFFN_ERR_INVALID, "moe_experts_grouped: null plan");
  if (R < 0 || expert_base < 0) return fail(MOEFFN_ERR_INVALID, "moe_experts_grouped: R=%d expert_base=%d", R, expert_base);
  if (R == 0) return MOEFFN_OK;
  if (rows == nullptr || row_expert == nullptr || d_out == nullptr)
    return fail(MOEFFN_ERR_INVALID, "moe_experts_grouped: null pointer");
  if (!aligned16(rows) || !aligned16(d_out))
    return fail(MOEFFN_ERR_INVALID, "moe_experts_grouped: rows/d_out not 16-byte aligned");
  if (p->E > kMaxExperts) return fail(MOEFFN_ERR_UNSUPPORTED, "moe_experts_grouped: %d experts (at most %d)", p->E, kMaxExperts);
  const int E = p->E, H = p->H, Ie = p->Ie, Is = p->Is;
  Carve c{nullptr};
  carve_moe(c, R, H, Ie, Is, E, 1);
  int rc = check_ws(ws, ws_bytes, c.off);
  if (rc != MOEFFN_OK) return rc;
  Carve cw{static_cast<char*>(ws)};
  const MoeWS w = carve_moe(cw, R, H, Ie, Is, E, 1);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  {
    PlaceArgs pa{row_expert, R, expert_base, E, w.offsets, w.perm, w.inv, w.union_list, w.n_union};
    ProfScope ps("place_rows", s);
    MOEFFN_CHECK_CUDA(launch_place_rows(pa, s), "row placement launch");
  }
  // Each row is one pair (k = 1): slot i of the grouped order reads row perm[i].
  int splits_r = 0, splits_s = 0;
  if ((rc = run_moe_phases(p, rows, R, 1, w, false, s, &splits_r, &splits_s)) != MOEFFN_OK) return rc;
  RowsFromSlotsArgs ra{w.d, splits_r, R, H, R, w.inv, d_out};
  ProfScope ps("rows_from_slots", s);
  MOEFFN_CHECK_CUDA(launch_rows_from_slots(ra, s), "split sum launch");
  return MOEFFN_OK;
}

size_t moe_combine_workspace_bytes(int M, int top_k) {
  if (M < 1 || top_k < 1) return 0;
  Carve c{nullptr};
  c.take<int>((size_t)M * top_k);
  return c.off;
}

int moe_combine(const float* d, const int32_t* perm, const float* topk_w, int M, int top_k, int H,
                const float* shared_d, const float* gate_logit, uint16_t* residual, void* ws, size_t ws_bytes,
                moeffn_stream_t stream) {
  g_last_error.clear();
  if (d == nullptr || perm == nullptr || topk_w == nullptr || residual == nullptr)
    return fail(MOEFFN_ERR_INVALID, "moe_combine: null pointer");
  if (shared_d != nullptr && gate_logit == nullptr)
    return fail(MOEFFN_ERR_INVALID, "moe_combine: shared_d needs gate_logit");
  if (M < 1 || top_k < 1 || top_k > kMaxTopK || H < 4 || H % 4 != 0)
    return fail(MOEFFN_ERR_INVALID, "moe_combine: M=%d top_k=%d H=%d (H a positive multiple of 4)", M, top_k, H);
  if (!aligned16(d) || !aligned16(residual) || (shared_d != nullptr && !aligned16(shared_d)))
    return fail(MOEFFN_ERR_INVALID, "moe_combine: d/shared_d/residual not 16-byte aligned");
  int rc = check_ws(ws, ws_bytes, moe_combine_workspace_bytes(M, top_k));
  if (rc != MOEFFN_OK) return rc;
  Carve cw{static_cast<char*>(ws)};
  int* inv = cw.take<int>((size_t)M * top_k);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  {
    InvertArgs ia{perm, M * top_k, inv};
    ProfScope ps("invert_perm", s);
    MOEFFN_CHECK_CUDA(launch_invert_perm(ia, s), "permutation inverse launch");
  }
  TailArgs t{};
  t.mode = TAIL_MOE;
  t.M = M;
  t.N = H;
  t.d = d;
  t.splits = 1;
  t.slots = M * top_k;
  t.d_s = shared_d;
  t.splits_s = shared_d != nullptr ? 1 : 0;
  t.gate_logit = gate_logit;
  t.w = topk_w;
  t.inv = inv;
  t.k = top_k;
  t.res = residual;
  ProfScope ps("tail_moe", s);
  MOEFFN_CHECK_CUDA(launch_tail(t, s), "moe tail launch");
  return MOEFFN_OK;
}

}  // extern "C"

namespace moeffn {
// Error reporting for the other translation units of the library.
int api_fail(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace moeffn
