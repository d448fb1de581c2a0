// kernels_simt.cu -- the bandwidth- and latency-bound steps of the layer
// (work-list build + offset validation, LayerNorm, gate, route builder,
// prediction head) and the fp32 build's CUDA-core GEMM / attention /
// combine.  All of them are warp- or block-level SIMT kernels with 16-byte
// vector access to rows of 512 elements.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace ptl {

// ------------------------------------------------------------------ rows
// One warp owns one row of 512 elements; lane l holds 16 of them.  For bf16
// rows the lane's elements are two 8-element (16-byte) chunks at l*8 and
// 256+l*8; for fp32 rows four 4-element chunks at l*4 + 128*i.
template <typename T>
struct Row16;

template <>
struct Row16<__nv_bfloat16> {
  __device__ static __forceinline__ int elem(int lane, int j) { return (j >> 3) * 256 + lane * 8 + (j & 7); }
  __device__ static __forceinline__ void load(const __nv_bfloat16* row, int lane, float (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(row + c * 256 + lane * 8));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        v[c * 8 + 2 * i] = f.x;
        v[c * 8 + 2 * i + 1] = f.y;
      }
    }
  }
  __device__ static __forceinline__ void store(__nv_bfloat16* row, int lane, const float (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint4 u;
      __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(v[c * 8 + 2 * i], v[c * 8 + 2 * i + 1]);
      *reinterpret_cast<uint4*>(row + c * 256 + lane * 8) = u;
    }
  }
};

template <>
struct Row16<float> {
  __device__ static __forceinline__ int elem(int lane, int j) { return (j >> 2) * 128 + lane * 4 + (j & 3); }
  __device__ static __forceinline__ void load(const float* row, int lane, float (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float4 f = __ldg(reinterpret_cast<const float4*>(row + c * 128 + lane * 4));
      v[c * 4 + 0] = f.x;
      v[c * 4 + 1] = f.y;
      v[c * 4 + 2] = f.z;
      v[c * 4 + 3] = f.w;
    }
  }
  __device__ static __forceinline__ void store(float* row, int lane, const float (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<float4*>(row + c * 128 + lane * 4) =
          make_float4(v[c * 4 + 0], v[c * 4 + 1], v[c * 4 + 2], v[c * 4 + 3]);
  }
};

// LayerNorm of the lane's 16 values of a 512-element row (two passes over
// registers: mean, then biased variance of the centred values).
// SMEM: g and b point to shared memory (plain loads) instead of global memory.
template <typename T, bool SMEM = false>
__device__ __forceinline__ void layer_norm16(float (&v)[16], const float* __restrict__ g,
                                             const float* __restrict__ b, int lane) {
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) s += v[j];
  const float mean = warp_sum(s) * (1.0f / D);
  float q = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    v[j] -= mean;
    q += v[j] * v[j];
  }
  const float rstd = rsqrtf(warp_sum(q) * (1.0f / D) + LN_EPS);
  // the lane's elements come in groups of 4 consecutive columns
#pragma unroll
  for (int qd = 0; qd < 4; ++qd) {
    const int c = Row16<T>::elem(lane, 4 * qd);
    const float4 g4 = SMEM ? *reinterpret_cast<const float4*>(g + c) : __ldg(reinterpret_cast<const float4*>(g + c));
    const float4 b4 = SMEM ? *reinterpret_cast<const float4*>(b + c) : __ldg(reinterpret_cast<const float4*>(b + c));
    v[4 * qd + 0] = v[4 * qd + 0] * rstd * g4.x + b4.x;
    v[4 * qd + 1] = v[4 * qd + 1] * rstd * g4.y + b4.y;
    v[4 * qd + 2] = v[4 * qd + 2] * rstd * g4.z + b4.z;
    v[4 * qd + 3] = v[4 * qd + 3] * rstd * g4.w + b4.w;
  }
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) ln_rows_kernel(const TI* __restrict__ x, const float* __restrict__ g,
                                                      const float* __restrict__ b, TO* __restrict__ y,
                                                      int T) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= T) return;
  float v[16];
  Row16<TI>::load(x + size_t(row) * D, lane, v);
  layer_norm16<TI>(v, g, b, lane);
  Row16<TO>::store(y + size_t(row) * D, lane, v);
}

// ------------------------------------------------------------- work list
// Validates cu_seqlens and lists the (user, query block) pairs of the
// jagged attention, heaviest first: a pair (u, b) needs b + 1 key blocks,
// so pairs are grouped by b in descending order (any order inside a group).
// One block of 1024 threads.
__device__ void block_suffix_exclusive(int32_t* a, int n) {
  // a[i] <- sum_{j > i} a[j] for i in [0, n), in chunks of blockDim taken from
  // the top so that the running carry flows downward; inside a chunk, thread
  // k holds a[top - k] and the chunk is scanned with warp shuffles and one
  // scan of the warp totals (three block barriers per chunk).
  __shared__ int32_t s_wtot[32];
  __shared__ int32_t s_carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
  if (threadIdx.x == 0) s_carry = 0;
  for (int top = n - 1; top >= 0; top -= blockDim.x) {
    const int i = top - int(threadIdx.x);
    const int32_t v = i >= 0 ? a[i] : 0;
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_wtot[warp] = incl;
    __syncthreads();  // (also orders the carry's previous update)
    if (warp == 0) {
      const int32_t tot = lane < nwarps ? s_wtot[lane] : 0;
      int32_t winc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, winc, o);
        if (lane >= o) winc += t;
      }
      s_wtot[lane] = winc - tot;  // exclusive prefix of the warp totals
    }
    __syncthreads();
    const int32_t carry = s_carry;
    if (i >= 0) a[i] = carry + s_wtot[warp] + incl - v;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry = carry + s_wtot[warp] + incl;
  }
  __syncthreads();
}

// The work list's arguments (one struct, passed by value).
struct WorklistArgs {
  const int32_t* cu;
  int U, T;
  int2* items;
  int32_t *item_count, *lvl_hist, *lvl_start, *lvl_fill;
  int max_levels, G;
  int4* ulist;
  int32_t *uoff, *ucnt, *err;
  AttnMask mask;
  int masked;
};

__device__ void worklist_body(const WorklistArgs& w);

__global__ void __launch_bounds__(1024) worklist_kernel(const WorklistArgs w) {
  pdl_wait();
  pdl_trigger();
  worklist_body(w);
}

// Slot of each kept token (mask[t] != 0) in ascending t, -1 for the others,
// and their count (n_pred, nullable): one block of 1024 threads in one pass,
// thread i owning the run of tokens [i * run, (i + 1) * run), the block's
// exclusive prefix of the runs' counts from warp shuffles and the 32 warp
// totals.  The compaction of the prediction head, taken ahead of it.
__device__ void head_slots_body(const uint8_t* __restrict__ mask, int32_t* __restrict__ slot,
                                int32_t* __restrict__ n_pred, int T_) {
  __shared__ int32_t s_warp[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int run = (T_ + 1023) / 1024;
  const int t0 = min(tid * run, T_), t1 = min(t0 + run, T_);
  int cnt = 0;
  for (int t = t0; t < t1; ++t) cnt += mask[t] ? 1 : 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int tot = s_warp[lane];
    int winc = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += v;
    }
    s_warp[lane] = winc - tot;  // exclusive prefix of the warp totals
    if (lane == 31 && n_pred) *n_pred = winc;
  }
  __syncthreads();
  int o = s_warp[warp] + incl - cnt;
  for (int t = t0; t < t1; ++t) slot[t] = mask[t] ? o++ : -1;
}

// The once-per-call prologue of the bf16 layer and stack: block 0 builds the
// attention work list (one block of 1024 threads, as worklist_kernel), block
// 1 takes the prediction head's output slots (with a mask), and the other
// blocks apply the first layer's LayerNorm1 to the input rows, one warp per row
// (the arithmetic of ln_rows_kernel); the three are independent.
__global__ void __launch_bounds__(1024) prologue_kernel(const WorklistArgs w, const __nv_bfloat16* __restrict__ x,
                                                        const float* __restrict__ g, const float* __restrict__ b,
                                                        __nv_bfloat16* __restrict__ y, int T,
                                                        const uint8_t* __restrict__ mask, int32_t* __restrict__ slot,
                                                        int32_t* __restrict__ n_pred) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0) {
    worklist_body(w);
    return;
  }
  if (blockIdx.x == 1) {
    if (mask) head_slots_body(mask, slot, n_pred, T);
    return;
  }
  // LayerNorm1 rows: one grid-wide warp stride (one wave of blocks, so no SM
  // runs two blocks back to back); each warp keeps its next P rows' loads in
  // flight as raw bf16 (8 registers a row) while it normalises the current
  // one, with gamma and beta read from shared memory.
  constexpr int P = 2;
  const int lane = threadIdx.x & 31;
  const int W = (gridDim.x - 2) * (blockDim.x >> 5);
  const int row = (blockIdx.x - 2) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  __shared__ __align__(16) float s_lg[D], s_lb[D];
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    s_lg[i] = g[i];
    s_lb[i] = b[i];
  }
  __syncthreads();
  if (row >= T) return;
  auto load_raw = [&](int r, uint4 (&u)[2]) {
    const uint4* src = reinterpret_cast<const uint4*>(x + size_t(r) * D);
    u[0] = __ldg(src + lane);
    u[1] = __ldg(src + 32 + lane);
  };
  uint4 raw[P][2];
#pragma unroll
  for (int i = 0; i < P; ++i)
    if (row + i * W < T) load_raw(row + i * W, raw[i]);
  for (int base = row; base < T; base += P * W) {
#pragma unroll
    for (int i = 0; i < P; ++i) {
      const int r = base + i * W;
      if (r < T) {
        float v[16];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[i][c]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(h[k]);
            v[c * 8 + 2 * k] = f.x;
            v[c * 8 + 2 * k + 1] = f.y;
          }
        }
        if (r + P * W < T) load_raw(r + P * W, raw[i]);
        layer_norm16<__nv_bfloat16, true>(v, s_lg, s_lb, lane);
        Row16<__nv_bfloat16>::store(y + size_t(r) * D, lane, v);
      }
    }
  }
}

// Shared-memory capacities of the work-list build: up to these sizes the
// offsets, the level counters and the items stay on chip (every count, scan
// and deal step is then a shared-memory access); larger inputs use the
// workspace arrays, with the same arithmetic.
constexpr int WL_SMEM_USERS = 2048;
constexpr int WL_SMEM_LEVELS = 1024;
constexpr int WL_SMEM_ITEMS = 2048;


__device__ void worklist_body(const WorklistArgs& w) {
  const int32_t* __restrict__ cu_g = w.cu;
  const int U = w.U, T = w.T;
  int2* __restrict__ items = w.items;
  int32_t* item_count = w.item_count;
  const int max_levels = w.max_levels, G = w.G;
  int4* __restrict__ ulist = w.ulist;
  int32_t* __restrict__ uoff = w.uoff;
  int32_t* __restrict__ ucnt = w.ucnt;
  int32_t* err = w.err;
  const AttnMask& mask = w.mask;
  const int masked = w.masked;
  __shared__ int s_bad;
  __shared__ int s_total;
  __shared__ int32_t s_cu[WL_SMEM_USERS + 1];
  __shared__ int32_t s_lstart[WL_SMEM_LEVELS], s_lfill[WL_SMEM_LEVELS];
  __shared__ int2 s_items[WL_SMEM_ITEMS];
  const int tid = threadIdx.x;
  const bool cu_s = U <= WL_SMEM_USERS, lv_s = max_levels + 1 <= WL_SMEM_LEVELS;
  // generic pointers: shared memory when the sizes fit, else the workspace
  const int32_t* cu = cu_s ? s_cu : cu_g;
  int32_t* lstart = lv_s ? s_lstart : w.lvl_start;
  int32_t* lfill = lv_s ? s_lfill : w.lvl_fill;
  if (tid == 0) {
    s_bad = (cu_g[0] != 0 || cu_g[U] != T) ? 1 : 0;
    s_total = 0;
  }
  if (cu_s)
    for (int i = tid; i <= U; i += blockDim.x) s_cu[i] = cu_g[i];
  for (int i = tid; i <= max_levels; i += blockDim.x) {
    lstart[i] = 0;  // first the number of users with exactly i query blocks
    lfill[i] = 0;
  }
  __syncthreads();
  for (int u = tid; u < U; u += blockDim.x)
    if (cu[u + 1] < cu[u]) s_bad = 1;
  __syncthreads();
  if (!s_bad && masked) {
    // contextual and candidate counts must fit in their user
    for (int u = tid; u < U; u += blockDim.x) {
      const int C = mask.ctx ? mask.ctx[u] : 0, N = mask.tgt ? mask.tgt[u] : 0;
      if (C < 0 || N < 0 || int64_t(C) + N > int64_t(cu[u + 1]) - cu[u]) s_bad = 2;
    }
    __syncthreads();
  }
  if (s_bad) {
    if (tid == 0) {
      *item_count = 0;
      set_error(err, s_bad == 2 ? PTL_ERR_BAD_MASK : PTL_ERR_BAD_OFFSETS);
    }
    for (int i = tid; i < 2 * G; i += blockDim.x) ucnt[i] = 0;
    return;
  }
  int local = 0;
  for (int u = tid; u < U; u += blockDim.x) {
    const int nb = (cu[u + 1] - cu[u] + ATT_BLK - 1) / ATT_BLK;
    if (nb > 0) atomicAdd(&lstart[nb], 1);
    local += nb;
  }
  atomicAdd(&s_total, local);
  __syncthreads();
  // lstart[b] <- #users with nb > b (pairs at level b) ...
  block_suffix_exclusive(lstart, max_levels + 1);
  // ... then the first slot of level b: sum over the deeper levels b' > b.
  block_suffix_exclusive(lstart, max_levels + 1);
  const bool it_s = s_total <= WL_SMEM_ITEMS;
  for (int u = tid; u < U; u += blockDim.x) {
    const int nb = (cu[u + 1] - cu[u] + ATT_BLK - 1) / ATT_BLK;
    for (int b = 0; b < nb; ++b) {
      const int slot = lstart[b] + atomicAdd(&lfill[b], 1);
      items[slot] = make_int2(u, b);
      if (it_s) s_items[slot] = make_int2(u, b);
    }
  }
  if (tid == 0) *item_count = s_total;
  __syncthreads();
  // The tensor-core attention's unit lists.  Unit u = 8 * item + head; CTA c
  // of the G-CTA grid takes units in snake order over the grid (0..G-1, then
  // G-1..0, ...: a mix of heavy and light units, the list being heaviest
  // first) and gives each to the stream (of two) with fewer key-block steps
  // so far.  Each (CTA, stream) list holds (s0, L, block, head) per unit in
  // order, so the kernel reads one independent descriptor per unit; with a
  // mask, (s0, L, block | head << 24, user) and a unit's steps are the key
  // blocks its mask leaves to walk.
  const int nunits = s_total * H;
  __shared__ int32_t s_off[2 * ATT_MAX_CTAS];
  for (int pass = 0; pass < 2; ++pass) {
    for (int c = tid; c < G; c += blockDim.x) {
      int acc0 = 0, acc1 = 0, n0 = 0, n1 = 0;
      for (int k = 0;; ++k) {
        const int u = k * G + ((k & 1) ? G - 1 - c : c);
        if (u >= nunits) break;
        const int2 it = it_s ? s_items[u >> 3] : items[u >> 3];
        int steps = it.y + 1;
        if (masked) {
          const int Lu = cu[it.x + 1] - cu[it.x];
          const int C = mask.ctx ? mask.ctx[it.x] : 0;
          const int Hs = Lu - (mask.tgt ? mask.tgt[it.x] : 0);
          int lo_key, hi_key;
          mask_key_range(it.y, Lu, C, Hs, mask, lo_key, hi_key);
          steps = hi_key / ATT_BLK - lo_key / ATT_BLK + 1;
        }
        const int to = acc0 <= acc1 ? 0 : 1;
        if (pass == 1) {
          const int s0 = cu[it.x];
          ulist[s_off[2 * c + to] + (to == 0 ? n0 : n1)] =
              masked ? make_int4(s0, cu[it.x + 1] - s0, it.y | ((u & 7) << 24), it.x)
                     : make_int4(s0, cu[it.x + 1] - s0, it.y, u & 7);
        }
        if (to == 0) {
          acc0 += steps;
          ++n0;
        } else {
          acc1 += steps;
          ++n1;
        }
      }
      if (pass == 0) {
        s_off[2 * c] = n0;
        s_off[2 * c + 1] = n1;
        ucnt[2 * c] = n0;
        ucnt[2 * c + 1] = n1;
      }
    }
    __syncthreads();
    if (pass == 0) {
      // exclusive prefix of the 2G list lengths, by warp 0: lane l owns a
      // contiguous run of entries
      if (tid < 32) {
        const int n = 2 * G, per = (n + 31) / 32;
        const int lo = tid * per, hi = min(n, lo + per);
        int sum = 0;
        for (int i = lo; i < hi; ++i) sum += s_off[i];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += v;
        }
        int run = incl - sum;
        for (int i = lo; i < hi; ++i) {
          const int len = s_off[i];
          s_off[i] = run;
          uoff[i] = run;
          run += len;
        }
      }
      __syncthreads();
    }
  }
}

// ------------------------------------------------------------------ gate
// One warp per token (grid-stride): LayerNorm2 of x1, the 8 gate logits in
// fp32 (w_gate staged once per block in shared memory), softmax, top-2 (ties
// to the lower index), renormalised weights.  Per-chunk route counts (128
// tokens = 256 routes per chunk, zeroed beforehand) are accumulated with
// atomics; the token's combine counters for the MoE are cleared.
constexpr int GATE_WARPS = 16;

__device__ __forceinline__ uint32_t sm_pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Sums a[0..7] over the warp and leaves expert (lane >> 2)'s total in a[0]:
// each exchange hands half of the remaining partial sums to the partner lane
// (4 + 2 + 1 shuffles), then two more butterflies finish the sum.
__device__ __forceinline__ float warp_reduce_scatter8(float (&a)[E], int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 16;
    const float send = hi ? a[i] : a[i + 4];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
    a[i] = (hi ? a[i + 4] : a[i]) + recv;
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 8;
    const float send = hi ? a[i] : a[i + 2];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
    a[i] = (hi ? a[i + 2] : a[i]) + recv;
  }
  {
    const bool hi = lane & 4;
    const float send = hi ? a[0] : a[1];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
    a[0] = (hi ? a[1] : a[0]) + recv;
  }
  a[0] += __shfl_xor_sync(0xffffffffu, a[0], 2);
  a[0] += __shfl_xor_sync(0xffffffffu, a[0], 1);
  return a[0];
}

// Stores the lane's 16 LayerNorm2 values (fp32 lane layout: 4 groups of 4
// consecutive columns at q*128 + lane*4) in the output dtype; a warp writes
// each group as one contiguous 256-byte (bf16) or 512-byte (fp32) segment.
__device__ __forceinline__ void store_row16_groups(__nv_bfloat16* row, int lane, const float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint2 u;
    u.x = sm_pack_bf16x2(v[4 * q], v[4 * q + 1]);
    u.y = sm_pack_bf16x2(v[4 * q + 2], v[4 * q + 3]);
    *reinterpret_cast<uint2*>(row + q * 128 + lane * 4) = u;
  }
}
__device__ __forceinline__ void store_row16_groups(float* row, int lane, const float (&v)[16]) {
  Row16<float>::store(row, lane, v);
}

// The gate for one token, by one warp: LayerNorm2 of the x1 row into v (the
// lane's 16 values in the fp32 lane layout: 4 groups of 4 consecutive columns
// at q*128 + lane*4), the 8 logits in fp32 against the staged gate weights,
// top-2 of the softmax (ties to the lower index) and the renormalised weights.
// Every lane returns the same e0, e1, w0, w1.
__device__ __forceinline__ void gate_token(const float* __restrict__ x1_row, const float* __restrict__ g,
                                           const float* __restrict__ b, const float* __restrict__ s_wg,
                                           const float* __restrict__ bg, int lane, float (&v)[16], int& e0,
                                           int& e1, float& w0, float& w1) {
  Row16<float>::load(x1_row, lane, v);
  layer_norm16<float>(v, g, b, lane);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 w4 = *reinterpret_cast<const float4*>(s_wg + e * D + q * 128 + lane * 4);
      s += v[4 * q] * w4.x + v[4 * q + 1] * w4.y + v[4 * q + 2] * w4.z + v[4 * q + 3] * w4.w;
    }
    acc[e] = s;
  }
  float mine = warp_reduce_scatter8(acc, lane) + (bg ? __ldg(bg + (lane >> 2)) : 0.f);
  float lg[E];
#pragma unroll
  for (int e = 0; e < E; ++e) lg[e] = __shfl_sync(0xffffffffu, mine, 4 * e);
  // softmax is monotonic, so the top-2 of p are the top-2 logits (ties to the
  // lower index), and the renormalised pair p0 / (p0 + p1), p1 / (p0 + p1)
  // depends only on their difference: w0 = 1 / (1 + t), w1 = t / (1 + t)
  // with t = exp(l1 - l0) <= 1.  Every lane evaluates the same values.
  e0 = 0;
  float l0 = lg[0];
#pragma unroll
  for (int e = 1; e < E; ++e)
    if (lg[e] > l0) {
      l0 = lg[e];
      e0 = e;
    }
  e1 = -1;
  float l1 = -INFINITY;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e != e0 && (e1 < 0 || lg[e] > l1)) {
      l1 = lg[e];
      e1 = e;
    }
  const float t = expf(l1 - l0);
  w0 = 1.0f / (1.0f + t);
  w1 = t * w0;
}

// Stages the gate weights [8][512] in shared memory; lane l later reads
// columns q*128 + 4l..4l+3, i.e. consecutive 16-byte words across the warp.
__device__ __forceinline__ void stage_gate_weights(float* s_wg, const float* __restrict__ wg) {
  for (int i = threadIdx.x; i < E * D / 4; i += blockDim.x)
    reinterpret_cast<float4*>(s_wg)[i] = __ldg(reinterpret_cast<const float4*>(wg) + i);
}

template <typename T>
__global__ void __launch_bounds__(GATE_WARPS * 32) gate_kernel(
    const float* __restrict__ x1, const float* __restrict__ g, const float* __restrict__ b,
    const float* __restrict__ wg, const float* __restrict__ bg, T* __restrict__ xn2,
    int32_t* __restrict__ idx, float* __restrict__ wout, int32_t* __restrict__ chunk_cnt, int T_) {
  __shared__ __align__(16) float s_wg[E * D];
  stage_gate_weights(s_wg, wg);
  __syncthreads();
  pdl_wait();  // x1 comes from the previous kernel
  pdl_trigger();  // dependents launch once this grid has passed its own wait
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int t = blockIdx.x * GATE_WARPS + warp; t < T_; t += gridDim.x * GATE_WARPS) {
    float v[16];
    int e0, e1;
    float w0, w1;
    gate_token(x1 + size_t(t) * D, g, b, s_wg, bg, lane, v, e0, e1, w0, w1);
    store_row16_groups(xn2 + size_t(t) * D, lane, v);
    if (lane == 0) {
      *reinterpret_cast<int2*>(idx + 2 * t) = make_int2(e0, e1);
      *reinterpret_cast<float2*>(wout + 2 * t) = make_float2(w0, w1);
      atomicAdd(&chunk_cnt[(t >> 7) * E + e0], 1);
      atomicAdd(&chunk_cnt[(t >> 7) * E + e1], 1);
    }
  }
}


// ------------------------------------------------------- gate + route
// The layer path's gate and route builder in one kernel (bf16 build).  A
// block of WARPS warps takes the next chunk of WARPS * GR_TPW tokens (a
// ticket, so chunks start in order); each warp runs the gate for GR_TPW
// consecutive tokens at once (the x1 rows of all of them in flight together;
// the LayerNorm2 and gate parameters, staged in shared memory before the
// wait for x1, serve all of them): LayerNorm2 in fp32, the 8 logits in fp32,
// the top-2 logits (ties to the lower index) and the renormalised weights.
// The chunk's routes are then ranked per expert (stable: ascending
// route id r = 2t + k), the chunk publishes its counts (flag 1) and sums the
// published counts of every earlier chunk (one thread per earlier chunk, in
// parallel; an earlier chunk's block took its ticket first, so it is running
// or done and will publish).  Expert e's rows start at e * cap (cap = T
// rounded up to 256 >= any expert's route count), so a route's row e * cap +
// (routes of e before it) needs no global totals: each warp writes pos[r]
// and stores each token's LayerNorm2 row (bf16) straight into both of its
// rows of xperm.  The last chunk also writes the expert tile list and the
// offsets.  Waits on predecessors are bounded (PTL_ERR_TIMEOUT).
// lb: [0] ticket, then per chunk 32 ints: [0] flag, [4..11] counts; all
// zero before the kernel.
template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) gate_route_kernel(
    const float* __restrict__ x1, const float* __restrict__ g, const float* __restrict__ b,
    const float* __restrict__ wg, const float* __restrict__ bg, int32_t* __restrict__ idx,
    float* __restrict__ wout, int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ xperm, int cap,
    int32_t* __restrict__ lb, int2* __restrict__ tiles, int32_t* __restrict__ meta,
    int32_t* __restrict__ moe_done, int max_tiles, int T_, int32_t* err) {
  constexpr int TOK = WARPS * GR_TPW;      // tokens of a chunk
  constexpr int ROUTES = 2 * TOK;
  constexpr int GROUPS = ROUTES / 32;      // 32-route groups ranked by one warp each
  static_assert(ROUTES % 32 == 0 && GROUPS <= WARPS, "route groups");
  __shared__ int s_chunk, s_e[ROUTES], s_rank[ROUTES], s_gcnt[GROUPS][E];
  __shared__ int s_cnt[E], s_excl[E], s_tot[E];
  __shared__ int s_red[WARPS][E];
  // the layer's LayerNorm2 and gate parameters, read before the wait for the
  // previous kernel (they are not its outputs) so that their first reads on
  // this SM do not sit on the path from x1 to the routes
  __shared__ __align__(16) float s_wg[E * D], s_g[D], s_b[D];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < E * D / 4; i += blockDim.x)
    reinterpret_cast<float4*>(s_wg)[i] = __ldg(reinterpret_cast<const float4*>(wg) + i);
  for (int i = threadIdx.x; i < D / 4; i += blockDim.x) {
    reinterpret_cast<float4*>(s_g)[i] = __ldg(reinterpret_cast<const float4*>(g) + i);
    reinterpret_cast<float4*>(s_b)[i] = __ldg(reinterpret_cast<const float4*>(b) + i);
  }
  const float bias_mine = bg ? __ldg(bg + (lane >> 2)) : 0.f;
  // The chunk ticket is taken before the wait for the previous kernel: the
  // counter was zeroed by a kernel (or the call's clear) that finished before
  // this grid could start, and the ticket orders only this grid's blocks
  // (every block that holds a ticket is resident and will publish, or
  // returns before any block looks back: on an error from earlier kernels
  // all of them do).
  if (threadIdx.x == 0) s_chunk = atomicAdd(lb, 1);
  pdl_wait();  // x1 comes from the previous kernel
  pdl_trigger();  // dependents launch once this grid has passed its own wait
  __syncthreads();
  const int c = s_chunk;
  const int nchunks = (T_ + TOK - 1) / TOK;
  const int t0 = c * TOK + warp * GR_TPW;  // this warp's first token
  // the x1 rows of the warp's tokens (fp32 lane layout: 4 groups of 4
  // consecutive columns at q*128 + lane*4), all loads issued together, and
  // the error word read beside them (they are in the workspace, valid to
  // read whatever an earlier kernel reported); the whole block then leaves
  // together if an earlier kernel reported an error
  float v[GR_TPW][16];
#pragma unroll
  for (int j = 0; j < GR_TPW; ++j) {
    const int t = t0 + j;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = t < T_ ? __ldg(reinterpret_cast<const float4*>(x1 + size_t(t) * D + q * 128 + lane * 4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      v[j][4 * q] = f.x;
      v[j][4 * q + 1] = f.y;
      v[j][4 * q + 2] = f.z;
      v[j][4 * q + 3] = f.w;
    }
  }
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = has_error(err) ? 1 : 0;
  __syncthreads();
  if (s_bad) return;
#pragma unroll
  for (int j = 0; j < GR_TPW; ++j) layer_norm16<float, true>(v[j], s_g, s_b, lane);
  // the 8 logits of every token: each weight load serves the warp's tokens;
  // the lane's 16 products summed as two interleaved fp32 partial sums (even
  // and odd columns) with paired FMAs, then added
  float acc[GR_TPW][E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    float4 w4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w4[q] = *reinterpret_cast<const float4*>(s_wg + e * D + q * 128 + lane * 4);
#pragma unroll
    for (int j = 0; j < GR_TPW; ++j) {
      uint64_t s2 = 0ull;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        s2 = sm100::f2_fma(sm100::f2_pack(v[j][4 * q], v[j][4 * q + 1]), sm100::f2_pack(w4[q].x, w4[q].y), s2);
        s2 = sm100::f2_fma(sm100::f2_pack(v[j][4 * q + 2], v[j][4 * q + 3]), sm100::f2_pack(w4[q].z, w4[q].w), s2);
      }
      float lo, hi;
      sm100::f2_unpack(s2, lo, hi);
      acc[j][e] = lo + hi;
    }
  }
  int e0s[GR_TPW], e1s[GR_TPW];
#pragma unroll
  for (int j = 0; j < GR_TPW; ++j) {
    const int t = t0 + j;
    const float mine = warp_reduce_scatter8(acc[j], lane) + bias_mine;
    float lg[E];
#pragma unroll
    for (int e = 0; e < E; ++e) lg[e] = __shfl_sync(0xffffffffu, mine, 4 * e);
    // softmax is monotonic: the top-2 of p are the top-2 logits (ties to the
    // lower index); w0 = 1 / (1 + t), w1 = t / (1 + t), t = exp(l1 - l0)
    int e0 = 0;
    float l0 = lg[0];
#pragma unroll
    for (int e = 1; e < E; ++e)
      if (lg[e] > l0) {
        l0 = lg[e];
        e0 = e;
      }
    int e1 = -1;
    float l1 = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (e != e0 && (e1 < 0 || lg[e] > l1)) {
        l1 = lg[e];
        e1 = e;
      }
    const float tt = expf(l1 - l0);
    const float w0 = 1.0f / (1.0f + tt);
    const float w1 = tt * w0;
    const bool valid = t < T_;
    e0s[j] = valid ? e0 : E;
    e1s[j] = valid ? e1 : E;
    if (valid && lane == 0) {
      *reinterpret_cast<int2*>(idx + 2 * t) = make_int2(e0, e1);
      *reinterpret_cast<float2*>(wout + 2 * t) = make_float2(w0, w1);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < GR_TPW; ++j) {
      s_e[2 * (warp * GR_TPW + j)] = e0s[j];
      s_e[2 * (warp * GR_TPW + j) + 1] = e1s[j];
    }
  }
  __syncthreads();
  // stable ranks inside each 32-route group and the groups' counts
  if (warp < GROUPS) {
    const int q = 32 * warp + lane;
    const int e = s_e[q];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    s_rank[q] = __popc(same & ((1u << lane) - 1u));
#pragma unroll
    for (int x = 0; x < E; ++x) {
      const unsigned bal = __ballot_sync(0xffffffffu, e == x);
      if (lane == x) s_gcnt[warp][x] = __popc(bal);
    }
  }
  __syncthreads();
  // publish this chunk's counts, then sum the counts of every earlier chunk
  int32_t* me = lb + 32 + 32 * c;
  if (threadIdx.x < E) {
    int n = 0;
#pragma unroll
    for (int gq = 0; gq < GROUPS; ++gq) n += s_gcnt[gq][threadIdx.x];
    s_cnt[threadIdx.x] = n;
    me[4 + threadIdx.x] = n;
  }
  // the block barrier orders the eight counts before thread 0's release
  // store, which makes them visible with the flag (cumulative release)
  __syncthreads();
  if (threadIdx.x == 0) sm100::st_release_gpu(me, 1);
  int part[E];
#pragma unroll
  for (int e = 0; e < E; ++e) part[e] = 0;
  for (int pc = threadIdx.x; pc < c; pc += blockDim.x) {
    const int32_t* pf = lb + 32 + 32 * pc;
    if (!sm100::wait_flag_at_least(pf, 1)) {
      set_error(err, PTL_ERR_TIMEOUT);
      break;
    }
    // the acquire load orders these after the flag
    const int4* src = reinterpret_cast<const int4*>(lb + 32 + 32 * pc + 4);
    const int4 v0 = __ldcg(src), v1 = __ldcg(src + 1);
    part[0] += v0.x;
    part[1] += v0.y;
    part[2] += v0.z;
    part[3] += v0.w;
    part[4] += v1.x;
    part[5] += v1.y;
    part[6] += v1.z;
    part[7] += v1.w;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int w = __reduce_add_sync(0xffffffffu, part[e]);
    if (lane == 0) s_red[warp][e] = w;
  }
  __syncthreads();
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    int excl = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) excl += s_red[w][e];
    s_excl[e] = excl;
    s_tot[e] = excl + s_cnt[e];
  }
  __syncthreads();
  // each token's two routes: rows e * cap + (routes of e before it); the
  // LayerNorm2 row goes out in bf16 (the layout of store_row16_groups)
#pragma unroll
  for (int j = 0; j < GR_TPW; ++j) {
    if (t0 + j >= T_) break;
    uint32_t vp[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) vp[i] = sm_pack_bf16x2(v[j][2 * i], v[j][2 * i + 1]);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = k == 0 ? e0s[j] : e1s[j];
      const int q = 2 * (warp * GR_TPW + j) + k;
      int rank = s_excl[e] + s_rank[q];
      for (int gq = 0; gq < (q >> 5); ++gq) rank += s_gcnt[gq][e];
      const int row = e * cap + rank;
      if (lane == 0) pos[2 * (t0 + j) + k] = row;
      __nv_bfloat16* dst = xperm + size_t(row) * D;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq)
        *reinterpret_cast<uint2*>(dst + qq * 128 + lane * 4) = make_uint2(vp[2 * qq], vp[2 * qq + 1]);
    }
  }
  if (c == nchunks - 1) {
    // the last chunk's inclusive prefix holds every expert's total
    int nt_before = 0;
    for (int e = 0; e < E; ++e) {
      const int nt = (s_tot[e] + MOE_BM - 1) / MOE_BM;
      for (int j = threadIdx.x; j < nt; j += blockDim.x) {
        tiles[nt_before + j] = make_int2(e, e * cap + j * MOE_BM);
        // the fused expert GEMMs' completion counters of both GEMMs
#pragma unroll
        for (int q = 0; q < MOE1_NT; ++q) moe_done[(nt_before + j) * MOE1_NT + q] = 0;
#pragma unroll
        for (int q = 0; q < MOE2_NT; ++q) moe_done[max_tiles * MOE1_NT + (nt_before + j) * MOE2_NT + q] = 0;
      }
      if (threadIdx.x == 0) meta[META_TILE0 + e] = nt_before;
      nt_before += nt;
    }
    if (threadIdx.x == 0) {
      meta[0] = nt_before;
      int off = 0;
      for (int e = 0; e < E; ++e) {
        meta[1 + e] = off;
        meta[10 + e] = e * cap;
        off += s_tot[e];
      }
      meta[1 + E] = off;
      meta[10 + E] = E * cap;
      meta[META_MOE_GO] = 0;
    }
  }
}

// Debug outputs of the fused path: perm (compact, stable) and expert_off from
// the rows gate_route_kernel assigned.  One thread per route.
__global__ void __launch_bounds__(256) route_debug_kernel(const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ pos,
                                                          const int32_t* __restrict__ meta, int cap,
                                                          int n_routes, int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ expert_off,
                                                          const int32_t* err) {
  pdl_wait();
  pdl_trigger();
  if (has_error(err)) return;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r <= E && blockIdx.x == 0 && expert_off) expert_off[r] = meta[1 + r];
  if (r >= n_routes || !perm) return;
  const int e = idx[r];
  perm[meta[1 + e] + (pos[r] - e * cap)] = r;
}

// Per-chunk route counts for a caller-supplied topk_idx (standalone route
// build); out-of-range expert ids set PTL_ERR_SHAPE and are skipped.
__global__ void __launch_bounds__(256) chunk_hist_kernel(const int32_t* __restrict__ idx, int n_routes,
                                                         int32_t* __restrict__ chunk_cnt, int32_t* err) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t s_hist[E];
  if (threadIdx.x < E) s_hist[threadIdx.x] = 0;
  __syncthreads();
  const int r = blockIdx.x * ROUTE_CHUNK + threadIdx.x;
  if (r < n_routes) {
    const int e = idx[r];
    if (e >= 0 && e < E)
      atomicAdd(&s_hist[e], 1);
    else
      set_error(err, PTL_ERR_SHAPE);
  }
  __syncthreads();
  if (threadIdx.x < E) chunk_cnt[blockIdx.x * E + threadIdx.x] = s_hist[threadIdx.x];
}

// ---------------------------------------------------------- route builder
// One block per chunk of 256 routes (one thread per route r = 2t + k).
// Stable counting sort: slot of r inside expert e = routes of e in earlier
// chunks + routes of e in earlier warps of this chunk + earlier lanes of
// this warp with the same expert.  Writes perm (compact slots), rowroute
// (padded slots: every expert's rows start on a MOE_BM-row boundary) and, in
// block 0, the padding (-1), the expert tile list and the offsets.  In the
// bf16 build (xn2 != NULL) it also copies each route's LayerNorm2 row to its
// padded slot of xperm, so the first expert GEMM reads its A rows by TMA
// (padding rows are left unwritten: their products land in padding rows of
// the expert outputs, which nothing reads).
constexpr int ROUTE_THREADS = 1024;  // the sort uses the first ROUTE_CHUNK threads, the row copy all

__global__ void __launch_bounds__(ROUTE_THREADS) route_kernel(
    const int32_t* __restrict__ idx, int n_routes, const int32_t* __restrict__ chunk_cnt,
    int32_t* __restrict__ perm, int32_t* __restrict__ pos, int32_t* __restrict__ rowroute,
    int2* __restrict__ tiles, int32_t* __restrict__ meta, int32_t* __restrict__ dbg_perm,
    int32_t* __restrict__ dbg_off, const __nv_bfloat16* __restrict__ xn2,
    __nv_bfloat16* __restrict__ xperm, const int32_t* err) {
  pdl_wait();
  pdl_trigger();
  constexpr int NW = ROUTE_THREADS / 32;
  __shared__ int32_t s_red[NW][2 * E];
  __shared__ int32_t s_pre[E], s_tot[E], s_off[E + 1], s_poff[E + 1];
  __shared__ int32_t s_wcnt[ROUTE_CHUNK / 32][E];
  __shared__ int32_t s_slot[ROUTE_CHUNK];  // padded slot of each route of the chunk (-1: none)
  if (has_error(err)) return;
  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_chunks = (n_routes + ROUTE_CHUNK - 1) / ROUTE_CHUNK;
  // routes of each expert in the chunks before this one (acc[0..E)) and in all
  // chunks (acc[E..2E))
  int acc[2 * E];
#pragma unroll
  for (int e = 0; e < 2 * E; ++e) acc[e] = 0;
  for (int cc = tid; cc < n_chunks; cc += ROUTE_THREADS) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int v = chunk_cnt[cc * E + e];
      acc[E + e] += v;
      if (cc < c) acc[e] += v;
    }
  }
#pragma unroll
  for (int e = 0; e < 2 * E; ++e) {
    int v = acc[e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_red[warp][e] = v;
  }
  if (tid < E) {
#pragma unroll
    for (int w = 0; w < ROUTE_CHUNK / 32; ++w) s_wcnt[w][tid] = 0;
  }
  __syncthreads();
  if (tid < 2 * E) {
    int v = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += s_red[w][tid];
    if (tid < E) s_pre[tid] = v; else s_tot[tid - E] = v;
  }
  __syncthreads();
  if (tid == 0) {
    s_off[0] = 0;
    s_poff[0] = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e + 1] = s_off[e] + s_tot[e];
      s_poff[e + 1] = s_poff[e] + (s_tot[e] + MOE_BM - 1) / MOE_BM * MOE_BM;
    }
  }
  // threads 0..ROUTE_CHUNK-1: one route each (whole warps, so the warp match is uniform)
  const bool sorter = tid < ROUTE_CHUNK;
  const int r = c * ROUTE_CHUNK + tid;
  bool valid = sorter && r < n_routes;
  int e = valid ? idx[r] : E;
  if (e < 0 || e >= E) {  // never index with an id outside [0, E)
    e = E;
    valid = false;
  }
  int rank = 0;
  if (sorter) {
    const unsigned same = __match_any_sync(0xffffffffu, e);
    rank = __popc(same & ((1u << lane) - 1u));
    if (valid && rank == 0) s_wcnt[warp][e] = __popc(same);
  }
  __syncthreads();
  if (sorter) {
    int slot = -1;
    if (valid) {
      int j = s_pre[e] + rank;
      for (int w = 0; w < warp; ++w) j += s_wcnt[w][e];
      perm[s_off[e] + j] = r;
      if (dbg_perm) dbg_perm[s_off[e] + j] = r;
      slot = s_poff[e] + j;
      rowroute[slot] = r;
      pos[r] = slot;
    }
    s_slot[tid] = slot;
  }
  if (xn2 != nullptr) {
    // every warp copies 8 of the chunk's 256 rows (1 KB each): lane l moves
    // 16-byte words l and l + 32 of each
    __syncthreads();
    constexpr int RPW = ROUTE_CHUNK / NW;  // rows per warp
#pragma unroll
    for (int h = 0; h < RPW; h += 4) {  // four rows (8 loads per lane) in flight
      uint4 v[4][2];
      int dst[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = warp * RPW + h + q;
        dst[q] = s_slot[k];
        const uint4* src = reinterpret_cast<const uint4*>(xn2 + size_t((c * ROUTE_CHUNK + k) >> 1) * D);
        v[q][0] = dst[q] >= 0 ? __ldg(src + lane) : make_uint4(0, 0, 0, 0);
        v[q][1] = dst[q] >= 0 ? __ldg(src + 32 + lane) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (dst[q] < 0) continue;
        uint4* d = reinterpret_cast<uint4*>(xperm + size_t(dst[q]) * D);
        d[lane] = v[q][0];
        d[32 + lane] = v[q][1];
      }
    }
  }
  if (c == 0) {
    __syncthreads();  // s_off / s_poff are written by thread 0
    for (int ee = 0; ee < E; ++ee) {
      for (int i = s_off[ee + 1] - s_off[ee] + tid; i < s_poff[ee + 1] - s_poff[ee]; i += ROUTE_THREADS)
        rowroute[s_poff[ee] + i] = -1;
      const int nt = (s_poff[ee + 1] - s_poff[ee]) / MOE_BM;
      for (int j = tid; j < nt; j += ROUTE_THREADS)
        tiles[s_poff[ee] / MOE_BM + j] = make_int2(ee, s_poff[ee] + j * MOE_BM);
    }
    if (tid == 0) meta[0] = s_poff[E] / MOE_BM;
    if (tid <= E) {
      meta[1 + tid] = s_off[tid];
      meta[10 + tid] = s_poff[tid];
      if (dbg_off) dbg_off[tid] = s_off[tid];
    }
  }
}

// ------------------------------------------------------------------ head
// The prediction head on one row held as 16 fp32 values per lane (the
// Row16 layout): LayerNorm_f, the dot product with w, + bias, clamp to
// +-LOGIT_CLAMP, sigmoid; lane 0 writes p[k].
__device__ __forceinline__ void head_row(float (&v)[16], const HeadArgs& hd, int lane, int k) {
  layer_norm16<__nv_bfloat16>(v, hd.g, hd.b, lane);
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) s += v[j] * __ldg(hd.w + Row16<__nv_bfloat16>::elem(lane, j));
  s = warp_sum(s) + (hd.bias ? __ldg(hd.bias) : 0.f);
  if (lane == 0) {
    const float z = fminf(fmaxf(s, -LOGIT_CLAMP), LOGIT_CLAMP);
    hd.probs[k] = 1.0f / (1.0f + expf(-z));
  }
}

template <typename T>
__global__ void __launch_bounds__(256) head_kernel(const T* __restrict__ h, const float* __restrict__ g,
                                                   const float* __restrict__ b,
                                                   const float* __restrict__ w,
                                                   const float* __restrict__ bias,
                                                   float* __restrict__ p, int T_) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T_) return;
  float v[16];
  Row16<T>::load(h + size_t(t) * D, lane, v);
  layer_norm16<T>(v, g, b, lane);
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) s += v[j] * __ldg(w + Row16<T>::elem(lane, j));
  s = warp_sum(s) + (bias ? __ldg(bias) : 0.f);
  if (lane == 0) {
    const float z = fminf(fmaxf(s, -LOGIT_CLAMP), LOGIT_CLAMP);
    p[t] = 1.0f / (1.0f + expf(-z));  // compacted afterwards
  }
}

// Keeps p[t] for the tokens with pred_mask[t] != 0, in ascending t.  One
// block of 1024 threads in one pass: thread i owns the contiguous run of
// tokens [i * run, (i + 1) * run), counts its kept tokens, the block takes
// the exclusive prefix of the counts (warp shuffles, then the 32 warp totals),
// and each thread writes its run's kept values in order.
__global__ void __launch_bounds__(1024) head_compact_kernel(const float* __restrict__ p,
                                                            const uint8_t* __restrict__ mask,
                                                            float* __restrict__ probs,
                                                            int32_t* __restrict__ n_pred, int T_) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t s_warp[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int run = (T_ + 1023) / 1024;
  const int t0 = min(tid * run, T_), t1 = min(t0 + run, T_);
  int cnt = 0;
  for (int t = t0; t < t1; ++t) cnt += mask[t] ? 1 : 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int tot = s_warp[lane];
    int winc = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, winc, o);
      if (lane >= o) winc += v;
    }
    s_warp[lane] = winc - tot;  // exclusive prefix of the warp totals
    if (lane == 31 && n_pred) *n_pred = winc;
  }
  __syncthreads();
  int o = s_warp[warp] + incl - cnt;
  for (int t = t0; t < t1; ++t)
    if (mask[t]) probs[o++] = p[t];
}

// ------------------------------------------------- fp32 build: CUDA cores
// C tile 64 x 64, K step 16, 256 threads with 4 x 4 outputs each.
// Modes: 0 = A rows direct, out = acc + bias (QKV projection)
//        1 = A rows direct, out = acc + bias + R (output projection + residual)
//        2 = A rows gathered through rowroute (token = route / 2), per-tile
//            expert weights, out = ReLU(acc + b1[e]) into the padded hidden rows
//        3 = A = padded hidden rows, per-tile expert weights, y[route] = acc + b2[e]
template <int MODE>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, int lda,
                                                       const float* __restrict__ W,
                                                       const float* __restrict__ bias,
                                                       const float* __restrict__ R,
                                                       float* __restrict__ C, int ldc, int M, int N,
                                                       int Kd, const int32_t* __restrict__ rowroute,
                                                       const int2* __restrict__ tiles,
                                                       const int32_t* __restrict__ meta,
                                                       const int32_t* err) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sA[16][64 + 4];
  __shared__ float sB[16][64 + 4];
  __shared__ int s_arow[64];
  if (has_error(err)) return;
  const int tid = threadIdx.x;
  int row0, expert = 0;
  if (MODE >= 2) {
    const int tile = blockIdx.x / (MOE_BM / 64);
    if (tile >= meta[0]) return;
    const int2 tl = tiles[tile];
    expert = tl.x;
    row0 = tl.y + (blockIdx.x % (MOE_BM / 64)) * 64;
  } else {
    row0 = blockIdx.x * 64;
  }
  const int n0 = blockIdx.y * 64;
  if (tid < 64) {
    const int m = row0 + tid;
    int ar;
    if (MODE == 2) {
      const int r = rowroute[m];
      ar = r < 0 ? -1 : r / K;
    } else if (MODE == 3) {
      ar = m;
    } else {
      ar = m < M ? m : -1;
    }
    s_arow[tid] = ar;
  }
  __syncthreads();
  const float* Wt = W + size_t(expert) * N * Kd;
  const int tr = tid / 16, tc = tid % 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < Kd; k0 += 16) {
    for (int i = tid; i < 64 * 16; i += 256) {
      const int r = i / 16, kk = i % 16;
      const int ar = s_arow[r];
      sA[kk][r] = ar >= 0 ? A[size_t(ar) * lda + k0 + kk] : 0.f;
      sB[kk][r] = (n0 + r < N) ? Wt[size_t(n0 + r) * Kd + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[kk][tr * 4 + i];
        bb[i] = sB[kk][tc * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = row0 + tr * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tc * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (MODE == 0) {
        if (m >= M) continue;
        C[size_t(m) * ldc + n] = v + (bias ? bias[n] : 0.f);
      } else if (MODE == 1) {
        if (m >= M) continue;
        C[size_t(m) * ldc + n] = v + (bias ? bias[n] : 0.f) + R[size_t(m) * ldc + n];
      } else if (MODE == 2) {
        v += bias ? bias[expert * N + n] : 0.f;
        C[size_t(m) * ldc + n] = fmaxf(v, 0.f);
      } else {
        const int r = rowroute[m];
        if (r < 0) continue;
        C[size_t(r) * ldc + n] = v + (bias ? bias[expert * N + n] : 0.f);
      }
    }
  }
}

// bf16 build: out[t] = (x1[t] + w[t][0] y(2t)) + w[t][1] y(2t+1) in fp32,
// rounded once; y(r) is row pos[r] of the padded per-route expert outputs
// (bf16).  One warp per token, 16-byte loads.  Inside a stack, the next
// layer's LayerNorm1 is applied to the rounded row as well (ln_g != NULL):
// xn = LN(out) with exactly the arithmetic of the standalone LayerNorm.
// STREAMED (after the fused expert GEMMs): launched as soon as the expert
// launch has started, the kernel does not wait for that grid to finish.  A
// warp first waits for the expert launch to have its inputs (meta[31], set
// by it once past its own dependency wait: pos and w, from the route
// builder, are then complete), then for the second-GEMM column tiles of both
// of its token's routes (their counters reach 2, one per CTA of the pair,
// released once the tiles' stores are complete), so the combine runs on the
// SMs the expert launch frees while its last tiles finish.  It waits for the
// expert grid at its end, so that its own completion still implies that of
// every earlier kernel.  Waits are bounded (PTL_ERR_TIMEOUT).
template <bool STREAMED>
__global__ void __launch_bounds__(256) combine_bf16_kernel(const __nv_bfloat16* __restrict__ ybuf,
                                                           const int32_t* __restrict__ pos,
                                                           const float* __restrict__ w,
                                                           const float* __restrict__ x1,
                                                           __nv_bfloat16* __restrict__ out, int T_,
                                                           const float* __restrict__ ln_g,
                                                           const float* __restrict__ ln_b,
                                                           __nv_bfloat16* __restrict__ xn,
                                                           int32_t* err, const int32_t* __restrict__ meta,
                                                           const int32_t* __restrict__ done2, const HeadArgs hd) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  bool ok = true;
  __shared__ int s_ok;
  static_assert(MOE2_NT == 2, "warp 0's lanes: 8 tokens x 2 routes x 2 column tiles");
  // The token's route rows, weights and x1 row come from kernels that
  // completed before the expert launch passed its dependency wait (this
  // grid starts only after that): every warp reads them first, before this
  // grid's own wait (or, streamed, while warp 0 waits for the expert tiles).
  int2 pr = make_int2(0, 0);
  float2 wt = make_float2(0.f, 0.f);
  float xr[16];
  if (t < T_) {
    pr = __ldcg(reinterpret_cast<const int2*>(pos) + t);
    wt = __ldcg(reinterpret_cast<const float2*>(w) + t);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f =
          __ldcg(reinterpret_cast<const float4*>(x1 + size_t(t) * D + Row16<__nv_bfloat16>::elem(lane, 4 * q)));
      xr[4 * q] = f.x;
      xr[4 * q + 1] = f.y;
      xr[4 * q + 2] = f.z;
      xr[4 * q + 3] = f.w;
    }
  }
  if (!STREAMED) pdl_wait();
  pdl_trigger();
  if (STREAMED) {
    // warp 0 waits for the whole block (the other warps sleep at the block
    // barrier, so that waiting blocks take few issue slots and little L2
    // bandwidth from the expert launch): first for the launch to have its
    // inputs, then lane l for column tile l % 2 of route (l / 2) % 2 of the
    // block's token l / 4
    if (warp == 0) {
      const uint32_t nap = 256;
      if (lane == 0 && !sm100::wait_flag_at_least(meta + META_MOE_GO, 1, sm100::kWaitLimitNs, nap)) ok = false;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && !has_error(err)) {
        const int tt = blockIdx.x * (blockDim.x >> 5) + (lane >> 2);
        if (tt < T_) {
          const int2 pr = __ldcg(reinterpret_cast<const int2*>(pos) + tt);
          const int slot = (lane & 2) ? pr.y : pr.x;
          const int cap = __ldcg(meta + 11) - __ldcg(meta + 10);  // expert e's rows start at e * cap
          const int e = slot / cap;
          const int mt = __ldcg(meta + META_TILE0 + e) + (slot - e * cap) / MOE_BM;
          if (!sm100::wait_flag_at_least(done2 + mt * MOE2_NT + (lane & 1), 2, sm100::kWaitLimitNs, nap))
            ok = false;
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) {
        if (!ok) set_error(err, PTL_ERR_TIMEOUT);
        // (an error from an earlier kernel also stops the block, read here
        // once for all its warps)
        s_ok = ok && !has_error(err) ? 1 : 0;
      }
    }
    __syncthreads();
    ok = s_ok != 0;
  }
  if (ok && t < T_ && (STREAMED || !has_error(err))) {
    if (ok) {
      float y0[16], y1[16], o[16];
      if (STREAMED) {
        // the rows were written by another kernel still running: read them
        // from L2 (the acquire loads above order these after the stores)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint4 u0 = __ldcg(reinterpret_cast<const uint4*>(ybuf + size_t(pr.x) * D + c * 256 + lane * 8));
          const uint4 u1 = __ldcg(reinterpret_cast<const uint4*>(ybuf + size_t(pr.y) * D + c * 256 + lane * 8));
          const __nv_bfloat162* p0 = reinterpret_cast<const __nv_bfloat162*>(&u0);
          const __nv_bfloat162* p1 = reinterpret_cast<const __nv_bfloat162*>(&u1);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f0 = __bfloat1622float2(p0[i]), f1 = __bfloat1622float2(p1[i]);
            y0[c * 8 + 2 * i] = f0.x;
            y0[c * 8 + 2 * i + 1] = f0.y;
            y1[c * 8 + 2 * i] = f1.x;
            y1[c * 8 + 2 * i + 1] = f1.y;
          }
        }
      } else {
        Row16<__nv_bfloat16>::load(ybuf + size_t(pr.x) * D, lane, y0);
        Row16<__nv_bfloat16>::load(ybuf + size_t(pr.y) * D, lane, y1);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = (xr[j] + wt.x * y0[j]) + wt.y * y1[j];
      Row16<__nv_bfloat16>::store(out + size_t(t) * D, lane, o);
      if (ln_g != nullptr) {
        // the values the next layer reads back: o rounded to bf16
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = __bfloat162float(__float2bfloat16_rn(o[j]));
        layer_norm16<__nv_bfloat16>(o, ln_g, ln_b, lane);
        Row16<__nv_bfloat16>::store(xn + size_t(t) * D, lane, o);
      } else if (hd.w != nullptr) {
        // the last layer of a stack: the prediction head on the stored
        // (bf16-rounded) row, for the tokens the prologue gave a slot
        const int k = __ldg(hd.slot + t);
        if (k >= 0) {
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __bfloat162float(__float2bfloat16_rn(o[j]));
          head_row(o, hd, lane, k);
        }
      }
    }
  }
  if (STREAMED) pdl_wait();
}

// fp32 build: out[t] = (x1[t] + w[t][0] * y[2t]) + w[t][1] * y[2t+1].
__global__ void __launch_bounds__(256) combine_f32_kernel(const float* __restrict__ y,
                                                          const float* __restrict__ w,
                                                          const float* __restrict__ x1,
                                                          float* __restrict__ out, int T_,
                                                          const int32_t* err) {
  pdl_wait();
  pdl_trigger();
  if (has_error(err)) return;
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= size_t(T_) * D) return;
  const size_t t = i / D, n = i % D;
  const float a = x1[i] + w[2 * t] * y[(2 * t) * D + n];
  out[i] = a + w[2 * t + 1] * y[(2 * t + 1) * D + n];
}

// Jagged causal attention on CUDA cores (fp32 build).  One block of 128
// threads per (user, query block, head) work item; thread i owns query row
// i of the block and runs an fp32 online softmax over the user's keys
// 0..q, staged 64 at a time in shared memory.
// MASKED: the keys walked and the keys visible follow the AttnMask (HSTU-style
// variants); otherwise keys 0 .. qi of the user (causal).
template <bool MASKED>
__global__ void __launch_bounds__(128) attn_f32_kernel(const float* __restrict__ qkv,
                                                       float* __restrict__ out,
                                                       const int32_t* __restrict__ cu,
                                                       const int2* __restrict__ items,
                                                       const int32_t* __restrict__ item_count,
                                                       const int32_t* err, const AttnMask mask) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sK[64][DH + 1];
  __shared__ float sV[64][DH + 1];
  if (has_error(err)) return;
  const int item = blockIdx.x / H, h = blockIdx.x % H;
  if (item >= *item_count) return;
  const int2 it = items[item];
  const int s0 = cu[it.x], L = cu[it.x + 1] - s0;
  const int qi = it.y * ATT_BLK + threadIdx.x;
  const bool valid = qi < L;
  float q[DH], o[DH];
  const float scale = 0.125f;
#pragma unroll
  for (int d = 0; d < DH; ++d) {
    q[d] = valid ? qkv[size_t(s0 + qi) * QKV_N + h * DH + d] * scale : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  int kbeg = 0, kend = min(L, (it.y + 1) * ATT_BLK);
  int C = 0, Hs = L;
  if (MASKED) {
    C = mask.ctx ? mask.ctx[it.x] : 0;
    Hs = L - (mask.tgt ? mask.tgt[it.x] : 0);
    int lo_key, hi_key;
    mask_key_range(it.y, L, C, Hs, mask, lo_key, hi_key);
    kbeg = lo_key / 64 * 64;
    kend = hi_key + 1;
  }
  for (int k0 = kbeg; k0 < kend; k0 += 64) {
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * DH; i += 128) {
      const int r = i / DH, d = i % DH;
      const int kj = k0 + r;
      sK[r][d] = kj < L ? qkv[size_t(s0 + kj) * QKV_N + D + h * DH + d] : 0.f;
      sV[r][d] = kj < L ? qkv[size_t(s0 + kj) * QKV_N + 2 * D + h * DH + d] : 0.f;
    }
    __syncthreads();
    if (!valid) continue;
    for (int r = 0; r < 64 && (MASKED ? k0 + r < kend : k0 + r <= qi); ++r) {
      if (MASKED && !mask_visible(qi, k0 + r, C, Hs, mask)) continue;
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < DH; ++d) s = fmaf(q[d], sK[r][d], s);
      const float mn = fmaxf(m, s);
      const float alpha = expf(m - mn);
      const float p = expf(s - mn);
      l = l * alpha + p;
#pragma unroll
      for (int d = 0; d < DH; ++d) o[d] = o[d] * alpha + p * sV[r][d];
      m = mn;
    }
  }
  if (!valid) return;
  const float inv = 1.0f / l;
#pragma unroll
  for (int d = 0; d < DH; ++d) out[size_t(s0 + qi) * D + h * DH + d] = o[d] * inv;
}

// ------------------------------------------------------ RepEncoder front end
// The batched embedding bag of the RepEncoder (cti2026 README, RepEncoder
// section) with its LayerNorm.  Blocks of 28 warps, one warp per slot, loop
// over tokens (token t = block, block + grid, ...), so each warp keeps its
// slot's LayerNorm scale and shift (its lane's 16 columns) in registers for
// the whole launch instead of re-reading 14336 x 8 bytes per token.  Per
// token a warp loads up to 32 of its bag's ids at once (coalesced), shuffles
// them to every lane and keeps DEPTH table rows in flight (each lane two
// 16-byte pieces of a 512-wide row, so a warp reads whole rows), summing in
// fp32 in bag order; the block then takes the mean and the biased variance
// of the token's 28 x 512 = 14336 sums (two passes over registers) and
// stores the normalised row in the output dtype.  An id outside its table or
// a malformed bag range sets PTL_ERR_BAD_IDS and contributes nothing.
constexpr int REP_WARPS = REP_SLOTS;

template <typename T>
__global__ void __launch_bounds__(REP_WARPS * 32)
    embag_ln_kernel(const __grid_constant__ RepTables tb, const int64_t* __restrict__ ids,
                    const int64_t* __restrict__ off, int64_t n_ids, int T_, const float* __restrict__ g,
                    const float* __restrict__ b, T* __restrict__ out, int32_t* err) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_red[REP_WARPS];
  __shared__ float s_stat;
  const int sl = threadIdx.x >> 5, lane = threadIdx.x & 31;  // warp = slot
  constexpr int NP = sizeof(T) == 2 ? 2 : 4;      // 16-byte pieces of a lane's 16 values
  constexpr int DEPTH = 1;                        // rows per step (the token loop keeps many warps busy)
  constexpr int ROW16 = D * int(sizeof(T)) / 16;  // 16-byte pieces per table row
  const int c0 = sl * D;
  float gs[16], bs[16];  // this lane's LayerNorm scale and shift, for every token
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int c = c0 + Row16<T>::elem(lane, j);
    gs[j] = __ldg(g + c);
    bs[j] = __ldg(b + c);
  }
  const uint4* table = static_cast<const uint4*>(tb.t[sl]);
  const int64_t vocab = tb.vocab[sl];
  bool bad = false;
  for (int t = blockIdx.x; t < T_; t += gridDim.x) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = 0.f;
    const int64_t b0 = off[size_t(t) * REP_SLOTS + sl], b1 = off[size_t(t) * REP_SLOTS + sl + 1];
    if (b0 < 0 || b1 < b0 || b1 > n_ids) {
      bad = true;
    } else {
      for (int64_t base = b0; base < b1; base += 32) {
        const int64_t i = base + lane;
        int64_t my = i < b1 ? __ldg(ids + i) : 0;
        const bool my_bad = i < b1 && (my < 0 || my >= vocab);
        if (__any_sync(0xffffffffu, my_bad)) bad = true;
        if (my_bad) my = -1;
        const int cnt = b1 - base < 32 ? int(b1 - base) : 32;
        for (int j = 0; j < cnt; j += DEPTH) {
          int64_t idq[DEPTH];
          uint4 raw[DEPTH][NP];
#pragma unroll
          for (int q = 0; q < DEPTH; ++q) idq[q] = __shfl_sync(0xffffffffu, my, j + q);
#pragma unroll
          for (int q = 0; q < DEPTH; ++q)
            if (j + q < cnt && idq[q] >= 0) {
              const uint4* row = table + size_t(idq[q]) * ROW16;
#pragma unroll
              for (int pc = 0; pc < NP; ++pc) raw[q][pc] = __ldg(row + pc * 32 + lane);
            }
#pragma unroll
          for (int q = 0; q < DEPTH; ++q)
            if (j + q < cnt && idq[q] >= 0) {
#pragma unroll
              for (int pc = 0; pc < NP; ++pc) {
                if constexpr (sizeof(T) == 2) {
                  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[q][pc]);
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h2[e]);
                    v[pc * 8 + 2 * e] += f.x;
                    v[pc * 8 + 2 * e + 1] += f.y;
                  }
                } else {
                  v[pc * 4 + 0] += __uint_as_float(raw[q][pc].x);
                  v[pc * 4 + 1] += __uint_as_float(raw[q][pc].y);
                  v[pc * 4 + 2] += __uint_as_float(raw[q][pc].z);
                  v[pc * 4 + 3] += __uint_as_float(raw[q][pc].w);
                }
              }
            }
        }
      }
    }
    // mean, then the biased variance of the centred values, over 14336
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) sum += v[j];
    sum = warp_sum(sum);
    if (lane == 0) s_red[sl] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = 0.f;
      for (int w = 0; w < REP_WARPS; ++w) a += s_red[w];
      s_stat = a * (1.0f / REP_W);
    }
    __syncthreads();
    const float mean = s_stat;
    float sq = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      v[j] -= mean;
      sq += v[j] * v[j];
    }
    sq = warp_sum(sq);
    __syncthreads();  // s_stat and s_red read by every thread before they are reused
    if (lane == 0) s_red[sl] = sq;
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = 0.f;
      for (int w = 0; w < REP_WARPS; ++w) a += s_red[w];
      s_stat = rsqrtf(a * (1.0f / REP_W) + LN_EPS);
    }
    __syncthreads();
    const float rstd = s_stat;
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = v[j] * rstd * gs[j] + bs[j];
    Row16<T>::store(out + size_t(t) * REP_W + c0, lane, v);
    __syncthreads();  // s_stat is rewritten by the next token
  }
  if (bad && lane == 0) set_error(err, PTL_ERR_BAD_IDS);
}

// --------------------------------------------------- FP8 (e4m3) operands
// Per-row e4m3 quantisation (one scale per row: s = max|row| / 448, 1 for an
// all-zero row; codes = the row divided by s, rounded to the nearest e4m3
// value, ties to even, saturating at +-448).  The scale and the quotient are
// IEEE float32 operations (correctly rounded division), so the codes are
// decided exactly as by a float32 restatement of the definition.  One warp
// per row, 16-byte accesses; cols is a multiple of 16.
template <typename T>
__global__ void __launch_bounds__(256) quant_rows_e4m3_kernel(const T* __restrict__ x, int64_t rows, int cols,
                                                              uint8_t* __restrict__ codes,
                                                              float* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += int64_t(gridDim.x) * (blockDim.x >> 5)) {
    const T* row = x + r * cols;
    float amax = 0.f;
    for (int c = lane * VEC; c < cols; c += 32 * VEC) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + c));
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int i = 0; i < VEC; ++i) amax = fmaxf(amax, fabsf(to_f32<T>(e[i])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (lane == 0) scales[r] = s;
    uint8_t* crow = codes + r * cols;
    for (int c = lane * 16; c < cols; c += 32 * 16) {
      float v[16];
#pragma unroll
      for (int h = 0; h < 16; h += VEC) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + c + h));
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int i = 0; i < VEC; ++i) v[h + i] = to_f32<T>(e[i]);
      }
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        w[q] = uint32_t(sm100::cvt_e4m3x2(__fdiv_rn(v[4 * q], s), __fdiv_rn(v[4 * q + 1], s))) |
               (uint32_t(sm100::cvt_e4m3x2(__fdiv_rn(v[4 * q + 2], s), __fdiv_rn(v[4 * q + 3], s))) << 16);
      *reinterpret_cast<uint4*>(crow + c) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// ------------------------------------------------------------- launchers
#define PTL_LAUNCH_CHECK() (cudaPeekAtLastError() == cudaSuccess ? 0 : -1)

int num_sms() {
  static PerDevice sms;
  const int n = sms.get([] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return -1;
    return v;
  });
  return n > 0 ? n : 148;
}

int launch_quant_rows_e4m3(const void* x, ptl_dtype dt, int64_t rows, int cols, uint8_t* codes, float* scales,
                           cudaStream_t st) {
  const int64_t want = (rows + 7) / 8;
  const int blocks = int(want < 8 * num_sms() ? want : 8 * num_sms());
  const int r = dt == PTL_BF16
                    ? launch_k(quant_rows_e4m3_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                               static_cast<const __nv_bfloat16*>(x), rows, cols, codes, scales)
                    : launch_k(quant_rows_e4m3_kernel<float>, dim3(blocks), dim3(256), 0, st,
                               static_cast<const float*>(x), rows, cols, codes, scales);
  return r != 0 ? -1 : PTL_LAUNCH_CHECK();
}

static WorklistArgs worklist_args(const int32_t* cu, int U, int T, const WsLayout& L, char* ws,
                                  const AttnMask* mask) {
  WorklistArgs w;
  w.cu = cu;
  w.U = U;
  w.T = T;
  w.items = reinterpret_cast<int2*>(ws + L.items);
  w.item_count = reinterpret_cast<int32_t*>(ws + L.item_count);
  w.lvl_hist = reinterpret_cast<int32_t*>(ws + L.lvl_hist);
  w.lvl_start = reinterpret_cast<int32_t*>(ws + L.lvl_start);
  w.lvl_fill = reinterpret_cast<int32_t*>(ws + L.lvl_fill);
  w.max_levels = int(L.max_levels);
  w.G = attn_grid(L.max_items, num_sms());
  w.ulist = reinterpret_cast<int4*>(ws + L.ulist);
  w.uoff = reinterpret_cast<int32_t*>(ws + L.uoff);
  w.ucnt = reinterpret_cast<int32_t*>(ws + L.ucnt);
  w.err = reinterpret_cast<int32_t*>(ws + L.err);
  w.mask = mask ? *mask : AttnMask{nullptr, nullptr, 1, 1, 0};
  w.masked = mask ? 1 : 0;
  return w;
}

int launch_worklist(const int32_t* cu, int U, int T, const WsLayout& L, char* ws, cudaStream_t st,
                    const AttnMask* mask) {
  if (launch_k(worklist_kernel, dim3(1), dim3(1024), 0, st, worklist_args(cu, U, T, L, ws, mask))) return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_prologue(const int32_t* cu, int U, int T, const WsLayout& L, char* ws, const void* x, const float* g,
                    const float* b, void* y, cudaStream_t st, const uint8_t* pred_mask, int32_t* n_pred) {
  // one block per SM (1024 threads of this kernel's register count fill
  // one): the work list, the head slots and up to SMs - 2 LayerNorm blocks
  const int ln_blocks = std::min((T + 31) / 32, std::max(1, num_sms() - 2));
  if (launch_k(prologue_kernel, dim3(2 + ln_blocks), dim3(1024), 0, st, worklist_args(cu, U, T, L, ws, nullptr),
               static_cast<const __nv_bfloat16*>(x), g, b, static_cast<__nv_bfloat16*>(y), T, pred_mask,
               reinterpret_cast<int32_t*>(ws + L.head_p), n_pred))
    return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_layernorm(const void* x, const float* g, const float* b, void* y, int T, ptl_dtype dt,
                     cudaStream_t st) {
  const int blocks = (T + 7) / 8;
  if (dt == PTL_BF16) {
    if (launch_k(ln_rows_kernel<__nv_bfloat16, __nv_bfloat16>, dim3(blocks), dim3(256), 0, st, 
        static_cast<const __nv_bfloat16*>(x), g, b, static_cast<__nv_bfloat16*>(y), T)) return -1;
  } else {
    if (launch_k(ln_rows_kernel<float, float>, dim3(blocks), dim3(256), 0, st, static_cast<const float*>(x), g, b,
                                                         static_cast<float*>(y), T)) return -1;
  }
  return PTL_LAUNCH_CHECK();
}

int launch_gate(const void* x1, const float* g, const float* b, const float* wg, const float* bg,
                void* xn2, int32_t* idx, float* w, int32_t* chunk_cnt, int T, ptl_dtype dt,
                cudaStream_t st) {
  // one token per warp: every token's row load is in flight at once (the
  // grid-stride loop only matters past 3 resident blocks per SM)
  int blocks = (T + GATE_WARPS - 1) / GATE_WARPS;
  if (blocks > 148 * 3 * 8) blocks = 148 * 3 * 8;
  if (dt == PTL_BF16) {
    if (launch_k(gate_kernel<__nv_bfloat16>, dim3(blocks), dim3(GATE_WARPS * 32), 0, st, 
        static_cast<const float*>(x1), g, b, wg, bg, static_cast<__nv_bfloat16*>(xn2), idx, w,
        chunk_cnt, T)) return -1;
  } else {
    if (launch_k(gate_kernel<float>, dim3(blocks), dim3(GATE_WARPS * 32), 0, st, static_cast<const float*>(x1), g, b, wg,
                                                           bg, static_cast<float*>(xn2), idx, w,
                                                           chunk_cnt, T)) return -1;
  }
  return PTL_LAUNCH_CHECK();
}

int launch_gate_route(const void* x1, const float* g, const float* b, const float* wg, const float* bg,
                      int T, const WsLayout& L, char* ws, cudaStream_t st) {
  // small chunks when they all fit one wave (one block per SM), so that
  // more SMs share the work; otherwise larger chunks, fewer to look back over
  const bool small = (T + GR_TOK_SMALL - 1) / GR_TOK_SMALL <= num_sms();
  auto go = [&](auto kernel, int warps, int tok) {
    return launch_k(kernel, dim3((T + tok - 1) / tok), dim3(warps * 32), 0, st, static_cast<const float*>(x1), g, b,
                    wg, bg, reinterpret_cast<int32_t*>(ws + L.idx), reinterpret_cast<float*>(ws + L.wgt),
                    reinterpret_cast<int32_t*>(ws + L.pos), reinterpret_cast<__nv_bfloat16*>(ws + L.xperm),
                    int(L.cap), reinterpret_cast<int32_t*>(ws + L.lb), reinterpret_cast<int2*>(ws + L.tiles),
                    reinterpret_cast<int32_t*>(ws + L.route_meta), reinterpret_cast<int32_t*>(ws + L.moe_done),
                    int(L.max_tiles), T, reinterpret_cast<int32_t*>(ws + L.err));
  };
  if (small ? go(gate_route_kernel<GR_WARPS_SMALL>, GR_WARPS_SMALL, GR_TOK_SMALL)
            : go(gate_route_kernel<GR_WARPS>, GR_WARPS, GR_TOK))
    return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_route_debug(int T, const WsLayout& L, const char* ws, int32_t* perm, int32_t* expert_off,
                       cudaStream_t st) {
  const int n = 2 * T;
  if (launch_k(route_debug_kernel, dim3((n + 255) / 256), dim3(256), 0, st,
               reinterpret_cast<const int32_t*>(ws + L.idx), reinterpret_cast<const int32_t*>(ws + L.pos),
               reinterpret_cast<const int32_t*>(ws + L.route_meta), int(L.cap), n, perm, expert_off,
               reinterpret_cast<const int32_t*>(ws + L.err)))
    return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_chunk_hist(const int32_t* idx, int T, int32_t* chunk_cnt, int32_t* err, cudaStream_t st) {
  const int n = 2 * T;
  if (launch_k(chunk_hist_kernel, dim3((n + ROUTE_CHUNK - 1) / ROUTE_CHUNK), dim3(ROUTE_CHUNK), 0, st, idx, n, chunk_cnt, err)) return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_route(const int32_t* idx, int T, const WsLayout& L, char* ws, int32_t* dbg_perm,
                 int32_t* dbg_off, const void* xn2, cudaStream_t st) {
  const int n = 2 * T;
  if (launch_k(route_kernel, dim3((n + ROUTE_CHUNK - 1) / ROUTE_CHUNK), dim3(ROUTE_THREADS), 0, st, 
      idx, n, reinterpret_cast<const int32_t*>(ws + L.chunk_cnt),
      reinterpret_cast<int32_t*>(ws + L.perm), reinterpret_cast<int32_t*>(ws + L.pos),
      reinterpret_cast<int32_t*>(ws + L.rowroute),
      reinterpret_cast<int2*>(ws + L.tiles), reinterpret_cast<int32_t*>(ws + L.route_meta),
      dbg_perm, dbg_off, static_cast<const __nv_bfloat16*>(xn2),
      xn2 ? reinterpret_cast<__nv_bfloat16*>(ws + L.xperm) : nullptr,
      reinterpret_cast<const int32_t*>(ws + L.err))) return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_head(const void* h, const ptl_head_weights* hw, const uint8_t* mask, float* probs,
                int32_t* n_pred, int T, ptl_dtype dt, const WsLayout& L, char* ws, cudaStream_t st) {
  // every token's probability into head_p, then the kept ones compacted
  float* p = reinterpret_cast<float*>(ws + L.head_p);
  const int blocks = (T + 7) / 8;
  const float* g = static_cast<const float*>(hw->lnf_g);
  const float* b = static_cast<const float*>(hw->lnf_b);
  const float* w = static_cast<const float*>(hw->w);
  const float* bias = static_cast<const float*>(hw->b);
  if (dt == PTL_BF16) {
    if (launch_k(head_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(h), g, b, w,
                 bias, p, T)) return -1;
  } else {
    if (launch_k(head_kernel<float>, dim3(blocks), dim3(256), 0, st, static_cast<const float*>(h), g, b, w, bias, p, T))
      return -1;
  }
  if (PTL_LAUNCH_CHECK() != 0) return -1;
  if (launch_k(head_compact_kernel, dim3(1), dim3(1024), 0, st, p, mask, probs, n_pred, T)) return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_gemm_f32(int mode, const float* A, int lda, const float* W, const float* bias,
                    const float* R, float* C, int ldc, int M, int N, int Kd, const WsLayout& L,
                    const char* ws, cudaStream_t st) {
  const int32_t* rr = reinterpret_cast<const int32_t*>(ws + L.rowroute);
  const int2* tiles = reinterpret_cast<const int2*>(ws + L.tiles);
  const int32_t* meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
  const int32_t* err = reinterpret_cast<const int32_t*>(ws + L.err);
  dim3 grid(mode >= 2 ? unsigned((MOE_BM / 64) * L.max_tiles) : unsigned((M + 63) / 64), unsigned((N + 63) / 64));
  int rc = 0;
  switch (mode) {
    case 0: rc = launch_k(gemm_f32_kernel<0>, dim3(grid), dim3(256), 0, st, A, lda, W, bias, R, C, ldc, M, N, Kd, rr, tiles, meta, err); break;
    case 1: rc = launch_k(gemm_f32_kernel<1>, dim3(grid), dim3(256), 0, st, A, lda, W, bias, R, C, ldc, M, N, Kd, rr, tiles, meta, err); break;
    case 2: rc = launch_k(gemm_f32_kernel<2>, dim3(grid), dim3(256), 0, st, A, lda, W, bias, R, C, ldc, M, N, Kd, rr, tiles, meta, err); break;
    default: rc = launch_k(gemm_f32_kernel<3>, dim3(grid), dim3(256), 0, st, A, lda, W, bias, R, C, ldc, M, N, Kd, rr, tiles, meta, err); break;
  }
  return rc != 0 ? -1 : PTL_LAUNCH_CHECK();
}

int launch_combine_bf16(const void* ybuf, const int32_t* pos, const float* w, const float* x1, void* out,
                        int T, const float* ln_g, const float* ln_b, void* xn, int32_t* err,
                        cudaStream_t st, const WsLayout* streamed_after, const char* ws, const HeadArgs* head) {
  const HeadArgs hd = head ? *head : HeadArgs{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  const auto* y = static_cast<const __nv_bfloat16*>(ybuf);
  auto* o = static_cast<__nv_bfloat16*>(out);
  auto* n = static_cast<__nv_bfloat16*>(xn);
  int rc;
  if (streamed_after) {
    const WsLayout& L = *streamed_after;
    const int32_t* meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
    const int32_t* done2 = reinterpret_cast<const int32_t*>(ws + L.moe_done) + L.max_tiles * MOE1_NT;
    rc = launch_k(combine_bf16_kernel<true>, dim3((T + 7) / 8), dim3(256), 0, st, y, pos, w, x1, o, T, ln_g, ln_b, n,
                  err, meta, done2, hd);
  } else {
    rc = launch_k(combine_bf16_kernel<false>, dim3((T + 7) / 8), dim3(256), 0, st, y, pos, w, x1, o, T, ln_g, ln_b, n,
                  err, static_cast<const int32_t*>(nullptr), static_cast<const int32_t*>(nullptr), hd);
  }
  if (rc) return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_combine_f32(const float* y, const float* w, const float* x1, float* out, int T,
                       const int32_t* err, cudaStream_t st) {
  const size_t n = size_t(T) * D;
  if (launch_k(combine_f32_kernel, dim3(unsigned((n + 255) / 256)), dim3(256), 0, st, y, w, x1, out, T, err)) return -1;
  return PTL_LAUNCH_CHECK();
}

int launch_embag_ln(const RepTables& tb, const int64_t* ids, const int64_t* off, int64_t n_ids, int T,
                    const float* g, const float* b, void* out, ptl_dtype dt, int32_t* err,
                    cudaStream_t st) {
  // blocks loop over tokens: one resident block per SM
  const int grid = T < num_sms() ? T : num_sms();
  if (dt == PTL_BF16) {
    if (launch_k(embag_ln_kernel<__nv_bfloat16>, dim3(grid), dim3(REP_WARPS * 32), 0, st, tb, ids, off, n_ids, T,
                 g, b, static_cast<__nv_bfloat16*>(out), err)) return -1;
  } else {
    if (launch_k(embag_ln_kernel<float>, dim3(grid), dim3(REP_WARPS * 32), 0, st, tb, ids, off, n_ids, T, g, b,
                 static_cast<float*>(out), err)) return -1;
  }
  return PTL_LAUNCH_CHECK();
}

int launch_attn_f32(const float* qkv, float* out, const int32_t* cu, const WsLayout& L,
                    const char* ws, cudaStream_t st, const AttnMask* mask) {
  const AttnMask m = mask ? *mask : AttnMask{nullptr, nullptr, 1, 1, 0};
  const auto args = [&](auto kern) {
    return launch_k(kern, dim3(unsigned(L.max_items * H)), dim3(128), 0, st, qkv, out, cu,
                    reinterpret_cast<const int2*>(ws + L.items),
                    reinterpret_cast<const int32_t*>(ws + L.item_count),
                    reinterpret_cast<const int32_t*>(ws + L.err), m);
  };
  if (mask ? args(attn_f32_kernel<true>) : args(attn_f32_kernel<false>)) return -1;
  return PTL_LAUNCH_CHECK();
}

// ------------------------------------------------------- wait self-test
// Waits on something that never happens, with the same bounded waits the
// layer's kernels use on their producers, so that the give-up path itself can
// be run: which == 0 waits on an mbarrier phase that no thread completes,
// which == 1 on a global flag (zeroed by the caller) that nothing raises.
// Each of the 32 threads gives up after limit_ns and the kernel records
// PTL_ERR_TIMEOUT in the error word; the context stays usable.
__global__ void __launch_bounds__(32) wait_selftest_kernel(int32_t* err, const int32_t* flag,
                                                           int which, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncwarp();
  const bool ok = which == 0 ? sm100::mbar_wait(&bar, 0, limit_ns)
                             : sm100::wait_flag_at_least(flag, 1, limit_ns);
  if (!ok) set_error(err, PTL_ERR_TIMEOUT);
}

int launch_wait_selftest(int32_t* err, const int32_t* flag, int which, uint64_t limit_ns,
                         cudaStream_t st) {
  if (launch_k(wait_selftest_kernel, dim3(1), dim3(32), 0, st, err, flag, which,
               static_cast<unsigned long long>(limit_ns))) return -1;
  return PTL_LAUNCH_CHECK();
}

}  // namespace ptl
