// attn_tc.cu -- jagged block-diagonal causal attention on tcgen05.
//
// A unit of work is (user u, 128-query block b, head h).  Units are listed on
// the device from cu_seqlens, heaviest first (block b needs b + 1 key blocks:
// the key loop stops at the diagonal block, so no [S,S] mask is built and no
// block above the diagonal is touched).  A persistent CTA per SM takes its
// units in snake order over the grid and splits them between two streams
// (each unit to the stream with fewer key-block steps so far); the work-list
// kernel writes each (CTA, stream) list of unit descriptors, so the CTA reads
// one independent descriptor per unit.  A stream is a sequence of steps
// (unit, key block kb).
// The producer and the MMA issuer serve the two streams independently (each
// polls both and advances whichever is ready), so a stream never waits for
// the other's softmax:
//
//   warp 0      TMA producer, straight from the packed qkv rows (128-byte
//               swizzle): the Q tile [128 x 64] of each stream's units
//               (double-buffered, so the next unit's Q loads while the
//               current unit runs), per step the K tile through a per-stream
//               2-deep ring (a slot frees when its QK^T is done) and the V
//               tile into the stream's single V buffer (freed by the
//               previous step's PV);
//   warps 1, 2  MMA issuers, one per stream: per step S = Q K^T (M=128, N =
//               the keys of this block rounded up to 16) into TMEM S[g], then
//               the previous step's O[g] += P V (M=128, N=64, K = its key
//               count; P is read from TMEM, V is the MN-major operand); a
//               unit's first PV overwrites O;
//   warps 3..18 softmax, four warpgroups, two per stream: thread r owns query
//               row r (TMEM lane r) of its stream's unit and half of the
//               block's 128 keys; per step it reads its half of the S row,
//               masks keys past its position and past the user, combines the
//               row maximum with the other half (shared memory + mbarrier),
//               keeps the running max m and its half's sum l in fp32 (base-2,
//               scale folded in) and writes P = exp2(s - m) as bf16 pairs into
//               TMEM.  m is raised lazily (only when a block's max exceeds it
//               by 2^8), and then its half of the O row in TMEM is rescaled in
//               place.  Before writing P it waits for the previous PV (the
//               stream's P buffer is single); at the end of a unit it stores
//               its half of O / l in bf16.
// Fully masked 32-key chunks of the diagonal block are skipped (their P is
// written as zeros); rows past the user end are computed but not stored; TMA
// zero-fills rows past T.  Every wait is bounded.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace ptl {
using namespace sm100;

constexpr int ATT_TILE_BYTES = ATT_BLK * DH * 2;  // 16 KB
// K ring stages per stream: a K tile is held until its QK^T is done and the
// next one must be loaded before the stream's next QK^T can start.
constexpr int ATT_KV_STAGES = 2;
// V buffers per stream: V of step n loads once the PV of step n - 2 is done.
constexpr int ATT_V_STAGES = 2;
// per stream: Q[2] + K[stages] + V[stages] (P lives in TMEM)
constexpr int ATT_SMEM_TILES = 2 * (2 + ATT_KV_STAGES + ATT_V_STAGES);
// the softmax halves' exchange: [parity][stream][half][row] maxima and sums
constexpr int ATT_XCHG_BYTES = 2 * (2 * 2 * 2 * 128 * 4);
constexpr int ATT_SMEM = ATT_SMEM_TILES * ATT_TILE_BYTES + ATT_XCHG_BYTES + 1024 + 512;  // + alignment, barriers
constexpr int ATT_THREADS = 608;  // producer, two MMA issuers, four softmax warpgroups (two per stream)

struct AttnUnit {
  int s0, L, b, h;
  int lo, hi;  // first and last key block the unit walks
  int C, Hs;   // masked variant: contextual tokens, first candidate (0 and L otherwise)
};

// One unit of a (CTA, stream) list written by the work-list kernel: (first
// token of the user, its length, query block, head); with a mask, (first
// token, length, block | head << 24, user), the user's contextual and
// candidate counts read from the mask and the key blocks derived from them.
template <bool MASKED>
__device__ __forceinline__ AttnUnit unit_from(const int4 d, const AttnMask& mk) {
  if constexpr (!MASKED) {
    return AttnUnit{d.x, d.y, d.z, d.w, 0, d.z, 0, d.y};
  } else {
    AttnUnit a;
    a.s0 = d.x;
    a.L = d.y;
    a.b = d.z & 0xFFFFFF;
    a.h = d.z >> 24;
    a.C = mk.ctx ? mk.ctx[d.w] : 0;
    a.Hs = a.L - (mk.tgt ? mk.tgt[d.w] : 0);
    int lo_key, hi_key;
    mask_key_range(a.b, a.L, a.C, a.Hs, mk, lo_key, hi_key);
    a.lo = lo_key / ATT_BLK;
    a.hi = hi_key / ATT_BLK;
    return a;
  }
}

// keys of block kb that exist for this user, rounded up to the MMA's 16
__device__ __forceinline__ int keys16(int L, int kb) {
  const int k = min(L - kb * ATT_BLK, ATT_BLK);
  return (k + 15) & ~15;
}

// One stream's position in the step sequence that the producer and the MMA
// issuers walk, plus (for the producer) whether the unit's Q load is issued.
// Each stream's next unit is looked up one unit ahead, so switching units
// does not wait on the unit list.  The two streams are held in named
// registers, never indexed by the stream number, so nothing lands in local
// memory.
struct StreamPos {
  int g;             // the stream (softmax warpgroup)
  int kb, n, uc;     // key block of the current unit, steps so far, units started
  bool live, nxt_live;
  AttnUnit u, nxt;   // current unit, the next one (looked up one unit ahead)
  const int4* list;  // this stream's units, in order
  const int4* first;  // its first two entries, read before the dependency wait (shared memory)
  int n_list, k_list;  // list length, next entry to read
  bool q_sent;       // producer: the current unit's Q tile load is issued
};

// The head of each stream's unit list: its offset, length and first two
// entries, read into shared memory before the kernel waits for the QKV
// projection (the work list was complete before this grid could start), so
// that no chain of dependent loads sits between that wait and the first tile
// loads.
struct AttnListHead {
  int off[2], cnt[2];
  int4 first[2][2];
};

// Both streams' step sequences as the producer and the MMA issuer walk them
// (`a` = stream 0, `b` = stream 1); each role advances a stream when that
// stream's next step can proceed.
template <bool MASKED>
struct AttnStepGen {
  const AttnMask& mk;
  __device__ explicit AttnStepGen(const AttnMask& m) : mk(m) {}
  __device__ void fetch_next(StreamPos& sp) {
    sp.nxt_live = sp.k_list < sp.n_list;
    if (sp.nxt_live) {
      const int4 d = sp.k_list < 2 ? sp.first[sp.k_list] : sp.list[sp.k_list];
      ++sp.k_list;
      sp.nxt = unit_from<MASKED>(d, mk);
    }
  }
  __device__ void init_stream(const int4* ulist, const AttnListHead& lh, int n_ok, StreamPos& sp, int g) {
    sp.g = g;
    sp.n = 0;
    sp.uc = 0;
    sp.list = ulist + lh.off[g];
    sp.first = lh.first[g];
    sp.n_list = n_ok ? lh.cnt[g] : 0;
    sp.k_list = 0;
    sp.q_sent = false;
    fetch_next(sp);
    sp.live = sp.nxt_live;
    sp.u = sp.nxt;
    sp.kb = sp.u.lo;
    if (sp.live) fetch_next(sp);
  }
  StreamPos a, b;
  __device__ void init(const int4* ulist, const AttnListHead& lh, int n_ok) {
    init_stream(ulist, lh, n_ok, a, 0);
    init_stream(ulist, lh, n_ok, b, 1);
  }
  // advances stream `sp` by one step
  __device__ void step(StreamPos& sp) {
    ++sp.n;
    if (++sp.kb > sp.u.hi) {
      ++sp.uc;
      sp.q_sent = false;
      sp.live = sp.nxt_live;
      sp.u = sp.nxt;
      sp.kb = sp.u.lo;
      if (sp.live) fetch_next(sp);
    }
  }
};


// MASKED: the HSTU-style variant (key blocks and visibility from the mask);
// otherwise block-diagonal causal.
template <bool MASKED>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const int4* __restrict__ ulist,
                   const int32_t* __restrict__ uoff, const int32_t* __restrict__ ucnt,
                   __nv_bfloat16* __restrict__ out, int32_t* __restrict__ err, const AttnMask mask,
                   const int list_early) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // per stream: Q[2 units], K[ATT_KV_STAGES steps], V[1 step], P[2 column blocks]
  uint8_t* sQ = smem;                                       // [stream][unit slot]
  uint8_t* sK = sQ + 2 * 2 * ATT_TILE_BYTES;                // [stream][stage]
  uint8_t* sV = sK + 2 * ATT_KV_STAGES * ATT_TILE_BYTES;    // [stream][stage]
  float* s_xm = reinterpret_cast<float*>(smem + ATT_SMEM_TILES * ATT_TILE_BYTES);  // [parity][stream][half][row]
  float* s_xl = s_xm + 2 * 2 * 2 * 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ATT_SMEM_TILES * ATT_TILE_BYTES + ATT_XCHG_BYTES);
  // Q is double-buffered (the next unit's Q loads while the current unit
  // runs); K is a ring whose slot frees once its QK^T is done; V (needed
  // only by the step's PV, a softmax step later) has one buffer per stream.
  uint64_t* q_full = bars;                            // [stream][unit slot]
  uint64_t* q_empty = bars + 4;                       // [stream][unit slot]
  uint64_t* k_full = bars + 8;                        // [stream][stage]
  uint64_t* k_empty = k_full + 2 * ATT_KV_STAGES;     // [stream][stage]
  uint64_t* v_full = k_empty + 2 * ATT_KV_STAGES;     // [stream][stage]
  uint64_t* v_empty = v_full + 2 * ATT_V_STAGES;      // [stream][stage]
  uint64_t* s_full = v_empty + 2 * ATT_V_STAGES;      // [stream]
  uint64_t* s_empty = s_full + 2;                 // [stream]
  uint64_t* p_full = s_full + 4;                  // [stream]
  uint64_t* pv_done = s_full + 6;                 // [stream]
  uint64_t* pv_empty = s_full + 8;                // [stream]
  uint64_t* x_bar = s_full + 10;                  // [stream] the two softmax halves meet
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 12);
  __shared__ int s_units;
  __shared__ AttnListHead s_lh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < 2 * ATT_V_STAGES; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 256);
      mbar_init(&p_full[i], 256);
      mbar_init(&pv_done[i], 1);
      mbar_init(&pv_empty[i], 256);
      mbar_init(&x_bar[i], 256);
    }
    for (int i = 0; i < 2 * ATT_KV_STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // this CTA's list heads (L2 reads).  list_early: the work list was written
  // by a kernel that had completed before the one this grid depends on
  // passed its own wait (the layer path: work list, QKV projection,
  // attention), so it is read before this grid's wait; otherwise after it.
  auto read_list_heads = [&]() {
    const int g = lane;
    const int off = __ldcg(uoff + 2 * blockIdx.x + g), cnt = __ldcg(ucnt + 2 * blockIdx.x + g);
    s_lh.off[g] = off;
    s_lh.cnt[g] = cnt;
    s_lh.first[g][0] = cnt > 0 ? __ldcg(ulist + off) : make_int4(0, 0, 0, 0);
    s_lh.first[g][1] = cnt > 1 ? __ldcg(ulist + off + 1) : make_int4(0, 0, 0, 0);
  };
  if (list_early && warp == 2 && lane < 2) read_list_heads();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();  // qkv and the error word come from earlier kernels (and the work list unless list_early)
  pdl_trigger();  // dependents launch once this grid has passed its own wait
  // n_ok = 0: an earlier kernel reported an error, no units.  On the layer
  // path (list_early) the error word is not read here: the lists are either
  // empty (the work list found bad offsets) or describe valid rows, so the
  // units run (on whatever an earlier failed kernel left) and the first
  // tile loads do not wait for that read.
  if (!list_early) {
    if (warp == 2 && lane < 2) read_list_heads();
    if (threadIdx.x == 0) s_units = has_error(err) ? 0 : 1;
    __syncthreads();
  }
  const int n_ok = list_early ? 1 : s_units;
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S[0] 0..127, S[1] 128..255, O[0] 256..319, O[1] 320..383,
  // P[0] 384..447, P[1] 448..511 (bf16 pairs)

  // The producer and the MMA issuer serve the two streams independently:
  // each polls both streams (non-blocking barrier tests: test_wait, which
  // never suspends the thread) and advances
  // whichever is ready, so neither stream waits for the other's softmax.
  // They give up (PTL_ERR_TIMEOUT) after a second without progress.
  if (warp == 0) {
    if (lane == 0) {
      AttnStepGen<MASKED> gen(mask);  // a = stream 0, b = stream 1 (never swapped here)
      gen.init(ulist, s_lh, n_ok);
      // V tiles wait in a small per-stream queue (row of the step's keys,
      // head): V of step n loads once the stream's PV of step n - 1 is done
      int vq0_row[2], vq0_col[2], vq1_row[2], vq1_col[2];  // [queue entry][stream]
      int vq_n[2] = {0, 0}, vq_len[2] = {0, 0};           // next V step, queued entries
      auto produce = [&](StreamPos& sp) -> bool {
        const int g = sp.g;
        bool prog = false;
        // the oldest queued V
        const int vs = g * ATT_V_STAGES + vq_n[g] % ATT_V_STAGES;
        if (vq_len[g] > 0 && mbar_test_wait(&v_empty[vs], ((vq_n[g] / ATT_V_STAGES) & 1) ^ 1)) {
          mbar_arrive_expect_tx(&v_full[vs], ATT_TILE_BYTES);
          tma_load_2d(sV + vs * ATT_TILE_BYTES, &tm_qkv, &v_full[vs], vq0_col[g], vq0_row[g]);
          ++vq_n[g];
          --vq_len[g];
          vq0_row[g] = vq1_row[g];
          vq0_col[g] = vq1_col[g];
          prog = true;
        }
        if (!sp.live || vq_len[g] == 2) return prog;
        const AttnUnit a = sp.u;
        const int qs = sp.uc & 1;  // the unit's Q slot
        if (sp.kb == a.lo && !sp.q_sent) {  // a new unit of stream g: its Q tile
          if (!mbar_test_wait(&q_empty[2 * g + qs], ((sp.uc >> 1) & 1) ^ 1)) return prog;
          mbar_arrive_expect_tx(&q_full[2 * g + qs], ATT_TILE_BYTES);
          tma_load_2d(sQ + (2 * g + qs) * ATT_TILE_BYTES, &tm_qkv, &q_full[2 * g + qs], a.h * DH,
                      a.s0 + a.b * ATT_BLK);
          sp.q_sent = true;
          prog = true;
        }
        // the step's K tile, once the slot's previous QK^T is done
        const int st = sp.n % ATT_KV_STAGES, use = sp.n / ATT_KV_STAGES;
        const int slot = g * ATT_KV_STAGES + st;
        if (!mbar_test_wait(&k_empty[slot], (use & 1) ^ 1)) return prog;
        mbar_arrive_expect_tx(&k_full[slot], ATT_TILE_BYTES);
        const int row = a.s0 + sp.kb * ATT_BLK;
        tma_load_2d(sK + slot * ATT_TILE_BYTES, &tm_qkv, &k_full[slot], D + a.h * DH, row);
        // queue its V
        if (vq_len[g] == 0) {
          vq0_row[g] = row;
          vq0_col[g] = 2 * D + a.h * DH;
        } else {
          vq1_row[g] = row;
          vq1_col[g] = 2 * D + a.h * DH;
        }
        ++vq_len[g];
        gen.step(sp);
        return true;
      };
      uint64_t t_prog = globaltimer_ns();
      while (gen.a.live || gen.b.live || vq_len[0] > 0 || vq_len[1] > 0) {
        bool prog = produce(gen.a);
        prog |= produce(gen.b);
        if (prog) {
          t_prog = globaltimer_ns();
        } else if (globaltimer_ns() - t_prog > kWaitLimitNs) {
          set_error(err, PTL_ERR_TIMEOUT);
          break;
        } else {
          __nanosleep(20);  // leave issue slots to the softmax warps while idle
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // MMA issuer of stream g = warp - 1 (one thread; the two streams' issuers
    // run independently): per step n, S(n) = Q K^T, then the previous step's
    // O += P V (a unit's first PV overwrites O, once warpgroup g has read the
    // previous unit's O).  The PV of step n - 1 is ready when S(n) can start
    // (both wait for the end of softmax step n - 1).
    if (lane == 0) {
      const int g = warp - 1;
      AttnStepGen<MASKED> gen(mask);
      StreamPos& sp = g == 0 ? gen.a : gen.b;
      gen.init_stream(ulist, s_lh, n_ok, sp, g);
      bool ok = true;
      int pvn = -1, pvk16 = 0, pvuc = 0;
      bool pvfirst = false;
      auto issue_pv = [&]() -> bool {
        if (pvn < 0) return true;
        if (!mbar_wait(&p_full[g], pvn & 1)) return false;
        if (pvfirst && !mbar_wait(&pv_empty[g], (pvuc & 1) ^ 1)) return false;
        const int vs = g * ATT_V_STAGES + pvn % ATT_V_STAGES;
        if (!mbar_wait(&v_full[vs], (pvn / ATT_V_STAGES) & 1)) return false;
        tc_fence_after();
        const uint32_t pt = tmem + 384 + 64 * g;  // P: 128 keys as bf16 pairs, 64 columns
        const uint32_t v0 = smem_u32(sV + vs * ATT_TILE_BYTES);
        const uint32_t d = tmem + 256 + 64 * g;
        constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 64, 0, 1);
        // the descriptors of the K slices differ only in the start-address
        // field (address / 16, no carry inside shared memory)
        const uint64_t dv = umma_desc_sw128(v0, 1024, 8192);
        const int nk = pvk16 / 16;
        for (int k = 0; k < nk; ++k)  // keys 16k..16k+15: P columns 8k..8k+7, V rows 2048 bytes on
          umma_bf16_ts(d, pt + 8 * k, dv + uint64_t(k * (2048 >> 4)), idesc_pv, k != 0 || !pvfirst);
        umma_commit(&pv_done[g]);
        umma_commit(&v_empty[vs]);
        pvn = -1;
        return true;
      };
      while (ok && sp.live) {
        const AttnUnit a = sp.u;
        const int kb = sp.kb, nn = sp.n;
        const int st = nn % ATT_KV_STAGES, use = nn / ATT_KV_STAGES;
        const int qs = sp.uc & 1;
        if ((kb == a.lo && !mbar_wait(&q_full[2 * g + qs], (sp.uc >> 1) & 1)) ||
            !mbar_wait(&k_full[g * ATT_KV_STAGES + st], use & 1) || !mbar_wait(&s_empty[g], (nn & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int k16 = keys16(a.L, kb);
        const uint32_t q0 = smem_u32(sQ + (2 * g + qs) * ATT_TILE_BYTES);
        const uint32_t k0 = smem_u32(sK + (g * ATT_KV_STAGES + st) * ATT_TILE_BYTES);
        const uint32_t idesc_qk = umma_idesc_bf16(128, k16);
        const uint64_t dq = umma_desc_sw128(q0, 1024), dk = umma_desc_sw128(k0, 1024);
#pragma unroll
        for (int k = 0; k < 4; ++k)  // K slices 32 bytes apart: +2 in the address field
          umma_bf16_ss(tmem + 128 * g, dq + uint64_t(2 * k), dk + uint64_t(2 * k), idesc_qk, k != 0);
        umma_commit(&s_full[g]);
        umma_commit(&k_empty[g * ATT_KV_STAGES + st]);
        if (kb == a.hi) umma_commit(&q_empty[2 * g + qs]);
        if (!issue_pv()) {
          ok = false;
          break;
        }
        pvn = nn;
        pvk16 = k16;
        pvfirst = kb == a.lo;
        pvuc = sp.uc;
        gen.step(sp);
      }
      if (ok) ok = issue_pv();
      if (!ok) set_error(err, PTL_ERR_TIMEOUT);
    }
  } else {
    // Softmax: four warpgroups, two per stream.  Warpgroup (g, h) (warps
    // 3 + 8g + 4h .. +3) handles keys 64h .. 64h + 63 of every S row of stream
    // g, column block h of P and columns 32h .. 32h + 31 of O; thread r <->
    // query row r <-> TMEM lane r.  The two halves of a row combine their
    // maxima (every step) and their sums (at a unit's end) through spare TMEM
    // columns, synchronised by a per-stream mbarrier (bounded waits).
    const int sw = (warp - 3) >> 2;
    const int g = sw >> 1, h = sw & 1;
    const int wq = warp & 3;
    const int r = 32 * wq + lane;
    const uint32_t lane_off = uint32_t(32 * wq) << 16;
    const uint32_t tS = tmem + 128 * g + 64 * h + lane_off;       // this half's 64 S columns
    const uint32_t tO = tmem + 256 + 64 * g + 32 * h + lane_off;  // this half's 32 O columns
    const uint32_t tP = tmem + 384 + 64 * g + 32 * h + lane_off;  // this half's 32 P columns (64 keys)
    // exchange slots: [parity][stream][half][row]
    auto xidx = [&](int par, int hh) { return ((par * 2 + g) * 2 + hh) * 128 + r; };
    const float c2 = 0.125f * 1.4426950408889634f;  // softmax scale * log2(e)
    // Running max m (base 2, scale folded in) of the row and this half's sum l.
    // O lives in TMEM and the PV products accumulate into it; m is raised (and
    // O, l rescaled) only when a block's max exceeds it by more than
    // RESCALE_LOG2, so P = exp2(s - m) stays below 2^RESCALE_LOG2 and O / l is
    // unchanged.  Both halves see the same maxima, so they keep the same m.
    constexpr float RESCALE_LOG2 = 8.f;
    float m = 0.f, l = 0.f;
    // the previous step of this stream: its PV may still be running
    int pn = -1;
    bool plast = false;
    float pl = 1.f;
    int pdst = -1;  // output row offset (elements) of this thread for the previous step's unit, or -1
    int nx = 0;     // exchanges of this stream so far
    bool ok = true;
    // both halves of the stream meet (every thread arrives, then waits)
    auto meet = [&]() -> bool {
      tc_fence_before();
      mbar_arrive(&x_bar[g]);
      const bool met = mbar_wait(&x_bar[g], nx & 1);
      ++nx;
      tc_fence_after();
      return met;
    };
    // waits for the previous step's PV; at a unit's end, stores this half's
    // columns of O / l and releases O for the next unit's first PV
    auto finish_prev = [&](float l_row) -> bool {
      if (!mbar_wait(&pv_done[g], pn & 1)) return false;
      tc_fence_after();
      if (plast) {
        const float inv = 1.0f / l_row;
        uint32_t raw[32];
        tmem_ld32(tO, raw);
        tmem_ld_wait();
        if (pdst >= 0) {
          uint4* dst = reinterpret_cast<uint4*>(out + pdst + 32 * h);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(raw[8 * q + 0]) * inv, __uint_as_float(raw[8 * q + 1]) * inv);
            u.y = pack_bf16x2(__uint_as_float(raw[8 * q + 2]) * inv, __uint_as_float(raw[8 * q + 3]) * inv);
            u.z = pack_bf16x2(__uint_as_float(raw[8 * q + 4]) * inv, __uint_as_float(raw[8 * q + 5]) * inv);
            u.w = pack_bf16x2(__uint_as_float(raw[8 * q + 6]) * inv, __uint_as_float(raw[8 * q + 7]) * inv);
            dst[q] = u;
          }
        }
        tc_fence_before();
        mbar_arrive(&pv_empty[g]);
      }
      return true;
    };
    int n = 0;  // steps of this stream
    const int4* list = ulist + s_lh.off[g];
    const int n_list = n_ok ? s_lh.cnt[g] : 0;
    int k_list = 0;
    AttnUnit nxt = k_list < n_list ? unit_from<MASKED>(s_lh.first[g][0], mask) : AttnUnit{0, 0, 0, 0, 0, 0, 0, 0};
    while (k_list < n_list && ok) {
      const AttnUnit a = nxt;
      ++k_list;
      if (k_list < n_list)  // look the next unit up
        nxt = unit_from<MASKED>(k_list < 2 ? s_lh.first[g][k_list] : list[k_list], mask);
      const int qi = a.b * ATT_BLK + r;   // query position inside the user
      const int qlim = min(qi, a.L - 1);  // keys 0..qlim are visible
      // masked variant: the row's visible keys as two intervals
      int va0 = 0, vb0 = -1, va1 = 0, vb1 = -1;
      if constexpr (MASKED) {
        if (qi < a.L) mask_row_intervals(qi, a.L, a.C, a.Hs, mask, va0, vb0, va1, vb1);
      }
      for (int kb = a.lo; kb <= a.hi; ++kb, ++n) {
        if (!mbar_wait(&s_full[g], n & 1)) { ok = false; break; }
        tc_fence_after();
        const int k16 = keys16(a.L, kb);
        const int kbase = kb * ATT_BLK;
        // 32-key chunks this warp needs: those inside the block's key count,
        // and on the diagonal block only chunks not wholly above the warp's
        // rows; this half owns chunks 2h and 2h + 1 (keys past qlim masked)
        const int nch = (k16 + 31) >> 5;
        const int nuse = (!MASKED && kb == a.b) ? min(nch, wq + 1) : nch;
        // masked variant: visibility of this half's 64 keys, one bit per key;
        // a warp whose rows see none of them skips the half (P written as 0)
        uint32_t vbits[2] = {0u, 0u};
        if constexpr (MASKED) {
          const int j0 = kbase + 64 * h;
          vbits[0] = interval_bits32(va0, vb0, j0) | interval_bits32(va1, vb1, j0);
          vbits[1] = interval_bits32(va0, vb0, j0 + 32) | interval_bits32(va1, vb1, j0 + 32);
        }
        const bool mine = 2 * h < nuse && (!MASKED || __any_sync(0xffffffffu, (vbits[0] | vbits[1]) != 0u));
        const int lim = qlim - (kbase + 64 * h);  // this half's keys i <= lim are visible
        // pass 1: this half's row maximum over the visible keys
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (mine) {
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {  // 32 columns per TMEM load
            uint32_t raw[32];
            tmem_ld32(tS + 32 * c, raw);
            tmem_ld_wait();
            const int lc = lim - 32 * c;
            if constexpr (MASKED) {
              const uint32_t bits = c ? vbits[1] : vbits[0];
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if ((bits >> i) & 1u) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(raw[i]));
            } else if (lc >= 31) {
#pragma unroll
              for (int i = 0; i < 32; i += 2)
                mx4[(i >> 1) & 3] = fmax3(mx4[(i >> 1) & 3], __uint_as_float(raw[i]), __uint_as_float(raw[i + 1]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (i <= lc) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(raw[i]));
            }
          }
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        // exchange the halves' maxima (and the previous step's sums)
        s_xm[xidx(n & 1, h)] = mx;
        if (!meet()) { ok = false; break; }
        const float xo = s_xm[xidx(n & 1, h ^ 1)];
        const float lo = (pn >= 0 && plast) ? s_xl[xidx(pn & 1, h ^ 1)] : 0.f;
        const float mblk = fmaxf(mx, xo) * c2;
        // the previous PV must be done before O is touched or P rewritten
        if (pn >= 0 && !finish_prev(pl + lo)) { ok = false; break; }
        if (kb == a.lo) {
          m = mblk;  // the unit's first PV overwrites O
          l = 0.f;
        } else if (__any_sync(0xffffffffu, mblk > m + RESCALE_LOG2)) {
          const float m_new = fmaxf(m, mblk);
          // masked variant: a row may have seen no visible key yet (m = -inf)
          const float alpha = (MASKED && m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
          uint32_t o[32];
          tmem_ld32(tO, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO, o);
          tmem_st_wait();
          l *= alpha;
          m = m_new;
        }
        // pass 2: this half's probabilities -> bf16 pairs in TMEM (P columns
        // 32h..32h+31); masked and skipped keys give p = 0
        if (mine) {
          uint64_t ls2[2] = {0ull, 0ull};  // paired partial sums
          const uint64_t c2x2 = f2_pack(c2, c2), negm = f2_pack(-m, -m);
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {  // keys 32c..32c+31 of the half: P columns 16c..16c+15
            uint32_t raw[32];
            tmem_ld32(tS + 32 * c, raw);
            tmem_ld_wait();
            const int lc = lim - 32 * c;
            const int lc_eff = lc >= 31 ? 31 : lc;
            uint32_t pk[16];
            const uint32_t bits = c ? vbits[1] : vbits[0];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const uint64_t xs = f2_fma(f2_pack(__uint_as_float(raw[i]), __uint_as_float(raw[i + 1])), c2x2, negm);
              float p0, p1;
              f2_unpack(xs, p0, p1);
              p0 = ex2_approx(p0);
              p1 = ex2_approx(p1);
              if constexpr (MASKED) {
                p0 = ((bits >> i) & 1u) ? p0 : 0.f;
                p1 = ((bits >> (i + 1)) & 1u) ? p1 : 0.f;
              } else if (lc < 31) {
                p0 = (i <= lc_eff) ? p0 : 0.f;
                p1 = (i + 1 <= lc_eff) ? p1 : 0.f;
              }
              ls2[(i >> 1) & 1] = f2_add(ls2[(i >> 1) & 1], f2_pack(p0, p1));
              pk[i >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tP + 16 * c, pk);
          }
          float s0, s1, s2, s3;
          f2_unpack(ls2[0], s0, s1);
          f2_unpack(ls2[1], s2, s3);
          l += (s0 + s1) + (s2 + s3);
        } else if (2 * h < nch) {
          uint32_t z[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) z[i] = 0u;
          tmem_st16(tP, z);
          tmem_st16(tP + 16, z);
        }
        tmem_st_wait();
        // this half's sum so far, for the other half at the unit's end
        s_xl[xidx(n & 1, h)] = l;
        // S is read and P written (and O rescaled): the next QK^T and this PV may start
        tc_fence_before();
        mbar_arrive(&s_empty[g]);
        mbar_arrive(&p_full[g]);
        pn = n;
        pl = l;
        plast = kb == a.hi;
        pdst = qi < a.L ? (a.s0 + qi) * D + a.h * DH : -1;
      }
    }
    if (ok && pn >= 0) {
      // the stream's last unit: the other half's sum, then O / l
      ok = meet();
      if (ok) ok = finish_prev(pl + s_xl[xidx(pn & 1, h ^ 1)]);
    }
    if (!ok) set_error(err, PTL_ERR_TIMEOUT);
  }
  __syncwarp();  // the single-lane roles rejoin their warps before the block barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool MASKED>
static int launch_attn_tc_t(const CUtensorMap& qkv_map, void* out, const WsLayout& L, char* ws,
                            cudaStream_t st, const AttnMask& mask, bool list_early) {
  static PerDevice configured;  // the shared-memory limit is a per-device kernel attribute
  if (configured.get([] {
        return cudaFuncSetAttribute(attn_tc_kernel<MASKED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    ATT_SMEM) == cudaSuccess
                   ? 1
                   : -1;
      }) < 0)
    return -1;
  // the work-list kernel laid out each CTA's units for this grid
  const int grid = attn_grid(L.max_items, num_sms());
  if (launch_k(attn_tc_kernel<MASKED>, dim3(grid), dim3(ATT_THREADS), ATT_SMEM, st, qkv_map,
               reinterpret_cast<const int4*>(ws + L.ulist), reinterpret_cast<const int32_t*>(ws + L.uoff),
               reinterpret_cast<const int32_t*>(ws + L.ucnt),
               static_cast<__nv_bfloat16*>(out), reinterpret_cast<int32_t*>(ws + L.err), mask,
               list_early ? 1 : 0) != 0)
    return -1;
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -1;
}

int launch_attn_tc(const CUtensorMap& qkv_map, void* out, const int32_t* cu, const WsLayout& L,
                   char* ws, cudaStream_t st, const AttnMask* mask, bool list_early) {
  (void)cu;
  if (mask) return launch_attn_tc_t<true>(qkv_map, out, L, ws, st, *mask, list_early);
  return launch_attn_tc_t<false>(qkv_map, out, L, ws, st, AttnMask{nullptr, nullptr, 1, 1, 0}, list_early);
}

}  // namespace ptl
