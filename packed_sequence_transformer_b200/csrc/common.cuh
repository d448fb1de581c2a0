// common.cuh -- layer constants, workspace layout and small device helpers
// shared by the kernels of the packed-sequence encoder layer.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/ptl.h"

namespace ptl {

constexpr int D = PTL_D_MODEL;     // 512
constexpr int H = PTL_N_HEADS;     // 8
constexpr int DH = PTL_D_HEAD;     // 64
constexpr int F = PTL_D_FF;        // 1024
constexpr int E = PTL_N_EXPERTS;   // 8
constexpr int K = PTL_TOP_K;       // 2
constexpr int QKV_N = 3 * D;       // 1536
constexpr int ATT_BLK = 128;       // query / key block of the jagged attention
constexpr int MOE_BM = 256;        // rows per expert tile (padding granule; one CTA pair's M)
constexpr int ROUTE_CHUNK = 256;   // routes per route-builder block (= 128 tokens)
// The fused gate + route kernel: GR_TPW tokens per warp, blocks of
// GR_WARPS_SMALL warps when every chunk fits one wave on the SMs (more SMs
// busy), else GR_WARPS warps (fewer chunks to look back over).
constexpr int GR_WARPS = 16;
constexpr int GR_WARPS_SMALL = 12;
constexpr int GR_TPW = 4;
constexpr int GR_TOK = GR_WARPS * GR_TPW;              // tokens per chunk (large blocks)
constexpr int GR_TOK_SMALL = GR_WARPS_SMALL * GR_TPW;  // tokens per chunk (small blocks)
constexpr int ATT_MAX_CTAS = 1024;  // bound on the persistent attention grid
constexpr int GEMM2_BN = 256;      // expert GEMM2 output columns per tile
constexpr int MOE1_NT = F / 256;   // expert GEMM1 column tiles per M tile (256 wide)
constexpr int MOE2_NT = D / 256;   // expert GEMM2 column tiles per M tile
// route_meta (int32 [32], written by the route builder): [0] M tiles, [1..9]
// expert route offsets, [10..18] expert row bases, [20..27] each expert's first
// M tile, [31] set (release) once the fused expert GEMMs have their inputs
constexpr int META_TILE0 = 20;
constexpr int META_MOE_GO = 31;
constexpr float LN_EPS = 1e-5f;
constexpr float LOGIT_CLAMP = 15.0f;

// Error word values are ptl_status codes; 0 = no error.
struct WsLayout {
  size_t err;         // int32 error word
  size_t items;       // int2 [max_items]   (user, query block) pairs, heaviest first
  size_t item_count;  // int32
  size_t lvl_hist;    // int32 [max_levels + 1]
  size_t lvl_start;   // int32 [max_levels + 1]
  size_t lvl_fill;    // int32 [max_levels + 1]
  size_t ulist;       // int4 [max_items * 8]  attention units per (CTA, stream): (s0, L, block, head)
  size_t uoff;        // int32 [2 * ATT_MAX_CTAS]  first entry of each (CTA, stream) list
  size_t ucnt;        // int32 [2 * ATT_MAX_CTAS]  entries of each (CTA, stream) list
  size_t xn;          // dt [T][512]    LayerNorm1 output
  size_t qkv;         // dt [T][1536]
  size_t attn;        // dt [T][512]
  size_t x1;          // f32 [T][512]   residual stream inside the layer
  size_t xn2;         // dt [T][512]
  size_t act0, act1;  // dt [T][512]    stack ping-pong
  size_t idx;         // int32 [T][2]
  size_t wgt;         // f32 [T][2]
  size_t chunk_cnt;   // int32 [n_chunks][8]
  size_t lb;          // int32 [32 + 32 * n_gchunks]  fused gate + route: ticket, per-chunk look-back state
  size_t moe_done;    // int32 [max_tiles][MOE1_NT] first-GEMM tiles done (CTAs), then
                      // int32 [max_tiles][MOE2_NT] second-GEMM tiles done (fused expert GEMMs)
  size_t perm;        // int32 [2T]
  size_t pos;         // int32 [2T]          route -> padded expert row
  size_t rowroute;    // int32 [padded_rows]   padded expert rows -> route (or -1)
  size_t tiles;       // int2 [max_tiles]     (expert, first padded row)
  size_t route_meta;  // int32 [32]: [0] n_tiles, [1..9] off, [10..18] first row of each expert
  size_t xperm;       // bf16 build: [padded_rows][512] LayerNorm2 rows in expert (padded) order
  size_t hbuf;        // dt [padded_rows][1024]  expert hidden rows (padded layout)
  size_t ybuf;        // per-route expert outputs awaiting the combine: bf16 build
                      // [padded_rows][512] bf16 in padded row order, fp32 build
                      // [2T][512] f32 in route order
  size_t head_p;      // f32 [T]            head probabilities before compaction
  size_t wl_end;      // end of the error word + work list (the no-alloc scratch holds these)
  size_t clear_end;   // end of the routing state that each call starts from zero
  size_t total;
  int64_t T;
  int32_t U;
  int64_t max_items, max_levels, n_chunks, max_tiles, padded_rows;
  int64_t n_gchunks;  // fused gate + route chunks (at most, GR_TOK_SMALL tokens each)
  int64_t cap;        // fused path: expert e's rows start at e * cap (T rounded up to MOE_BM)
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The persistent attention grid: one CTA per SM, at most one per unit (the
// work-list kernel lays out each CTA's units for exactly this grid).
__host__ inline int attn_grid(int64_t max_items, int num_sms) {
  int64_t g = max_items * H;
  if (g > num_sms) g = num_sms;
  if (g > ATT_MAX_CTAS) g = ATT_MAX_CTAS;
  return g < 1 ? 1 : int(g);
}

__host__ inline bool make_layout(int64_t T, int32_t U, ptl_dtype dt, WsLayout* L) {
  if (T < 0 || T >= (int64_t(1) << 31) || U < 1) return false;
  if (dt != PTL_F32 && dt != PTL_BF16) return false;
  const size_t es = dt == PTL_BF16 ? 2 : 4;
  L->T = T;
  L->U = U;
  const int64_t nonempty_users = U < T ? U : T;
  L->max_items = (T + ATT_BLK - 1) / ATT_BLK + nonempty_users + 1;
  L->max_levels = (T + ATT_BLK - 1) / ATT_BLK + 1;
  L->n_chunks = (2 * T + ROUTE_CHUNK - 1) / ROUTE_CHUNK + 1;
  L->max_tiles = (2 * T + MOE_BM - 1) / MOE_BM + E + 1;
  L->n_gchunks = (T + GR_TOK_SMALL - 1) / GR_TOK_SMALL + 1;  // the smaller chunks
  L->cap = (T + MOE_BM - 1) / MOE_BM * MOE_BM;
  // expert rows: compact-padded (route builder) or at fixed e * cap (fused path)
  L->padded_rows = 2 * T + E * MOE_BM;
  if (E * L->cap > L->padded_rows) L->padded_rows = E * L->cap;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), 256);
    return at;
  };
  L->err = take(256);
  L->items = take(sizeof(int2) * L->max_items);
  L->item_count = take(4);
  L->lvl_hist = take(4 * (L->max_levels + 1));
  L->lvl_start = take(4 * (L->max_levels + 1));
  L->lvl_fill = take(4 * (L->max_levels + 1));
  L->ulist = take(16 * L->max_items * H);
  L->uoff = take(4 * 2 * ATT_MAX_CTAS);
  L->ucnt = take(4 * 2 * ATT_MAX_CTAS);
  L->wl_end = o;  // error word + attention work list
  L->chunk_cnt = take(4 * L->n_chunks * E);
  L->lb = take(4 * (32 + 32 * L->n_gchunks));
  L->moe_done = take(4 * L->max_tiles * (MOE1_NT + MOE2_NT));
  L->clear_end = o;  // [0, clear_end) is cleared by one memset per call
  L->xn = take(es * T * D);
  L->qkv = take(es * T * QKV_N);
  L->attn = take(es * T * D);
  L->x1 = take(4 * T * D);
  L->xn2 = take(es * T * D);
  L->act0 = take(es * T * D);
  L->act1 = take(es * T * D);
  L->idx = take(4 * T * K);
  L->wgt = take(4 * T * K);
  L->perm = take(4 * 2 * T);
  L->pos = take(4 * 2 * T);
  L->rowroute = take(4 * L->padded_rows);
  L->tiles = take(sizeof(int2) * L->max_tiles);
  L->route_meta = take(4 * 32);
  L->xperm = take(dt == PTL_BF16 ? 2 * L->padded_rows * D : 0);
  L->hbuf = take(es * L->padded_rows * F);
  L->ybuf = take(dt == PTL_BF16 ? 2 * L->padded_rows * D : 4 * 2 * T * D);
  L->head_p = take(4 * T);
  L->total = o;
  return true;
}

// ---------------------------------------------------------------- RepEncoder
constexpr int REP_SLOTS = 28;
constexpr int REP_W = REP_SLOTS * D;  // 14336 values per token
// The 28 embedding tables (device pointers, [vocab][512] in the build dtype)
// and their row counts, passed by value to the embedding-bag kernel.
struct RepTables {
  const void* t[REP_SLOTS];
  int64_t vocab[REP_SLOTS];
};

// ---------------------------------------------------------------- masks
// HSTU-style attention masks (cry-daniel/recsys README, HSTU attention mask
// logic).  A user's L tokens are laid out [contextual][historical][candidate]:
// the first C are contextual, the candidates start at Hs = L - N.  Key j is
// visible to query i (positions inside the user, j < L) when
//   - causal ? j <= i : always, or both are contextual (i < C and j < C);
//   - and, for a candidate key (j >= Hs), i is a candidate of the same group
//     (groups of `group` candidates counted from Hs);
//   - and, with window > 0, |i - j| < window.
// Every query sees itself, so no row of a valid batch is fully masked.
struct AttnMask {
  const int32_t* ctx;  // [U] contextual tokens per user, or nullptr (none)
  const int32_t* tgt;  // [U] candidate tokens per user, or nullptr (none)
  int32_t causal;      // 1: causal base rule; 0: every key of the user
  int32_t group;       // candidates per group (>= 1)
  int32_t window;      // > 0: sliding window; <= 0: none
};

__host__ __device__ __forceinline__ bool mask_visible(int i, int j, int C, int Hs, const AttnMask& m) {
  bool v = m.causal ? j <= i : true;
  v = v || (i < C && j < C);
  if (j >= Hs) v = v && i >= Hs && (i - Hs) / m.group == (j - Hs) / m.group;
  if (m.window > 0) v = v && (i > j ? i - j : j - i) < m.window;
  return v;
}

// The keys visible to query i under the mask, as two intervals [a0, b0] and
// [a1, b1] of positions (an interval with a > b is empty): a non-candidate
// row sees [0 .. (causal ? (contextual ? C - 1 : i) : L - 1)] below the
// first candidate; a candidate row sees [0, Hs - 1] and, second, its own
// group up to itself (causal) or to the group's end.  Both are then cut to
// the window.  The same set as mask_visible, for every i < L.
__host__ __device__ __forceinline__ void mask_row_intervals(int i, int L, int C, int Hs, const AttnMask& m,
                                                   int& a0, int& b0, int& a1, int& b1) {
  a0 = 0;
  a1 = 1;
  b1 = 0;  // empty
  if (i < Hs) {
    int hi = m.causal ? (i < C ? C - 1 : i) : L - 1;
    b0 = hi < Hs - 1 ? hi : Hs - 1;
  } else {
    b0 = Hs - 1;
    const int g0 = Hs + (i - Hs) / m.group * m.group;
    const int rest = L - 1 - g0;  // keys of the user from g0 on, less one
    a1 = g0;
    b1 = m.causal ? i : g0 + (m.group - 1 < rest ? m.group - 1 : rest);
  }
  if (m.window > 0) {
    const int wl = i - m.window + 1, wh = i + m.window - 1;
    if (wl > a0) a0 = wl;
    if (wh < b0) b0 = wh;
    if (wl > a1) a1 = wl;
    if (wh < b1) b1 = wh;
  }
}

// Bits k (0..31) set where j0 + k lies in [a, b].
__host__ __device__ __forceinline__ uint32_t interval_bits32(int a, int b, int j0) {
  int lo = a - j0, hi = b - j0 + 1;  // bits [lo, hi)
  lo = lo > 0 ? lo : 0;
  hi = hi < 32 ? hi : 32;
  if (hi <= lo) return 0u;
  const uint32_t below_hi = hi >= 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u);
  return below_hi & ~((1u << lo) - 1u);
}

// Keys [lo_key, hi_key] that hold every key visible to some query of block b
// (queries q0 .. q1 of the user): the range the key loop walks.
__host__ __device__ __forceinline__ void mask_key_range(int b, int L, int C, int Hs, const AttnMask& m,
                                               int& lo_key, int& hi_key) {
  const int q0 = b * ATT_BLK;
  const int q1 = q0 + ATT_BLK - 1 < L - 1 ? q0 + ATT_BLK - 1 : L - 1;
  int hi = m.causal ? q1 : L - 1;
  if (q0 < C && C - 1 > hi) hi = C - 1;    // contextual rows see the whole context
  if (q1 < Hs && Hs - 1 < hi) hi = Hs - 1;  // no candidate row: no candidate key
  int lo = 0;
  if (m.window > 0) {
    lo = q0 - m.window + 1 > 0 ? q0 - m.window + 1 : 0;
    if (q1 + m.window - 1 < hi) hi = q1 + m.window - 1;
  }
  lo_key = lo;
  hi_key = hi;
}

// ---------------------------------------------------------------- device
// Programmatic dependent launch.  Every kernel of the library is launched so
// that the next kernel in the stream may start its prologue while this one
// runs: each kernel waits for its own predecessor to complete (and its writes
// to be visible) before it reads anything the predecessor produced, and only
// then allows its dependents to launch (trigger).  So at most one kernel runs
// ahead: a persistent kernel's CTAs cannot occupy SMs while a kernel two
// places earlier still needs them.  Every kernel executes the wait on every
// path, so completion stays transitive along the stream.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_error(int32_t* err, int32_t code) {
  atomicCAS(err, 0, code);
}
__device__ __forceinline__ bool has_error(const int32_t* err) {
  return *reinterpret_cast<const volatile int32_t*>(err) != 0;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace ptl
