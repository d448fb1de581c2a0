// gemm_tc.cu -- tcgen05 GEMMs of the layer (bf16 in, fp32 accumulate in TMEM).
//
// D = A B^T with A [M][K] and B = W [N][K] (nn.Linear layout), both K-major
// in shared memory with the 128-byte swizzle, on CTA pairs: a cluster of two
// CTAs (two SMs) computes 256 x BN output tiles with M=256 tcgen05.mma
// (cta_group::2).  Each pair is persistent and walks a static round-robin list
// of tiles.  CTA c of the pair holds rows m0 + 128c of A and rows
// n0 + c*BN/2 of B in its own shared memory; both CTAs' loads count on CTA 0's
// `full` barrier; CTA 0's single MMA thread issues the MMAs, which read both
// CTAs' operands and write each CTA's 128 rows of D into its own TMEM; its
// commits arrive on both CTAs' barriers.  Two TMEM accumulators (2 x BN
// columns) let the epilogue of one tile run while the tensor core works on
// the next.  Warp roles in each CTA:
//   warp 0      TMA producer: one elected thread streams 64-wide K slices of
//               A and B through a STAGES-deep ring of shared-memory buffers;
//   warp 1      allocates TMEM (both CTAs); in CTA 0 one thread issues the
//               MMAs (M=256, N=BN, K=16), commits each ring stage back to both
//               producers and each finished accumulator to both epilogues;
//   warps 2..9  epilogue: each thread owns one accumulator row (TMEM lane)
//               and one half of the tile's columns (two warps per TMEM lane
//               quarter), reads them with tcgen05.ld, releases the
//               accumulator on CTA 0 (one arrival per warp), applies the
//               fused epilogue and stages the tile for a TMA bulk-tensor
//               store.
// Sharing B across the pair halves B's shared-memory traffic per output: at
// this problem size the GEMMs are bound by L2 -> SM operand traffic, so the
// tile shape is chosen for bytes per FLOP.
// Modes:
//   QKV   qkv = xn Wqkv^T + b_qkv                         (A by TMA)
//   OUT   x1  = x + attn Wo^T + b_o, kept in fp32         (A by TMA)
//   MOE1  H[row] = ReLU(xperm[row] W1[e]^T + b1[e])       (A by TMA: the route
//         builder copies each route's LayerNorm2 row to its padded row)
//   MOE2  Y[row] = H[row] W2[e]^T + b2[e]                 (A by TMA)
//   FP8   out = (xq wq^T) * sx[row] * sw[col] + b         (e4m3 codes, kind::f8f6f4;
//         a 128-byte K slice holds 128 codes, so K steps by 128)
//         (per-route expert outputs in padded row order, bf16; the top-2
//         weighted combine + residual runs in combine_bf16_kernel)
// The expert GEMMs' rows are padded per expert to 256 (one pair tile never
// straddles two experts).
// Every wait is bounded; a timeout sets PTL_ERR_TIMEOUT and unwinds.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace ptl {
using namespace sm100;

struct GemmTcParams {
  int M;                         // rows of A (dense modes)
  int N_total;                   // output columns (per expert in the MoE modes)
  int num_kb;                    // K / 64
  int n_tiles_dense;             // dense modes: ceil(M / 256) * (N_total / BN)
  const float* bias;             // [N] or [E][N]; may be NULL
  const __nv_bfloat16* resid;    // OUT: x (row stride 512)
  __nv_bfloat16* out;            // output rows
  float* out_f32;                // OUT: x1 in fp32
  int ldo;                       // output row stride (elements)
  const int2* tiles;             // (expert, first padded row) per 256-row M tile
  const int32_t* meta;           // [0] = number of M tiles
  int max_mt;                    // capacity of `tiles` (entries)
  int32_t* zero_ptr;             // cleared by the grid once the predecessor is done (may be NULL)
  int zero_n;
  // MOE12 (both expert GEMMs in one launch): the second GEMM's width, bias
  // and per-M-tile completion counters of the first GEMM (zero at launch)
  int N2;
  const float* bias2;
  int32_t* done;
  int32_t* err;
  // FP8: per-row scales of A (rows of the output) and of B (its columns)
  const float* sx;
  const float* sw;
  // weights of later kernels to bring into L2 while this one waits for its
  // inputs (16-byte aligned, sizes multiples of 16; may be NULL)
  const void* pf_ptr[2];
  size_t pf_bytes[2];
};

enum { G_QKV = 0, G_OUT = 1, G_MOE1 = 2, G_MOE2 = 3, G_MOE12 = 4, G_FP8 = 5 };
// expert modes: rows padded per expert, tiles from the route builder's list
__host__ __device__ constexpr bool is_moe(int mode) { return mode == G_MOE1 || mode == G_MOE2 || mode == G_MOE12; }

// Warps per CTA: producer, MMA issuer, and 8 epilogue warps (two per TMEM
// lane quarter, each taking half of the tile's columns).
constexpr int GEMM_EPI_WARPS = 8;
constexpr int GEMM_STORE_WARP = 2 + GEMM_EPI_WARPS;  // issues the bf16 tiles' TMA stores
constexpr int GEMM_THREADS = 64 + 32 * GEMM_EPI_WARPS + 32;

// Shared-memory plan: the operand ring, the output staging tile and the
// tile's bias slice.
template <int BN, int MODE>
struct PairCfg {
  static constexpr int OUT_ELEM = MODE == G_OUT ? 4 : 2;
  static constexpr int BOX_COLS = 128 / OUT_ELEM;
  // columns staged (and stored) at a time: the fp32 output goes out in
  // parts of 64 columns through two 32 KB
  // buffers, so that a part is staged while the previous one is stored
  static constexpr int PART = MODE == G_OUT ? 64 : BN;
  // bf16 tiles 256 wide stage in two rounds of 128 columns (one 64-column
  // box per column half) through a 32 KB buffer: two more operand stages fit
  static constexpr bool HALF_STG = MODE != G_OUT && BN == 256;
  static constexpr int STAGING = HALF_STG ? 128 * 128 * 2 : (MODE == G_OUT ? 2 : 1) * 128 * PART * OUT_ELEM;
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = (BN / 2) * 64 * 2;
  // FP8: the bias and the weight rows' scales, double-buffered by tile (the
  // other modes read the bias through L1)
  static constexpr int BIAS = MODE == G_FP8 ? 2 * 2 * BN * 4 : 0;
  static constexpr int USABLE = 232448 - 1024 - 256 - 64;
  static constexpr int STAGES_FIT = (USABLE - STAGING - BIAS) / (A_BYTES + B_BYTES);
  static constexpr int STAGES = STAGES_FIT > 10 ? 10 : STAGES_FIT;
  static constexpr int SMEM = STAGES * (A_BYTES + B_BYTES) + STAGING + BIAS + 1024 + 256;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static_assert(2 * BN <= 512 && BN % 32 == 0 && B_BYTES % 1024 == 0, "tile width");
  static_assert(STAGES >= 2, "operand ring too small");
};

// Pair tile `tile` -> (expert, first row of the pair's 256 rows, first column).
// For MOE12 the tiles of the first expert GEMM come first (M tiles x F/BN),
// then those of the second (M tiles x D/BN); `second` tells them apart and
// `mt` is the tile's M tile.
template <int BN, int MODE>
__device__ __forceinline__ void decode_pair_tile(const GemmTcParams& p, int tile, int n_mt, int& expert,
                                                 int& m0, int& n0, bool& second, int& mt,
                                                 const int2* tl_known = nullptr, int known_mt = -1) {
  second = false;
  int nN = p.N_total / BN;
  if (MODE == G_MOE12 && tile >= n_mt * nN) {
    tile -= n_mt * nN;
    nN = p.N2 / BN;
    second = true;
  }
  mt = tile / nN;
  n0 = (tile - mt * nN) * BN;
  if (is_moe(MODE)) {
    const int2 tl = (tl_known && mt == known_mt) ? *tl_known : p.tiles[mt];
    expert = tl.x;
    m0 = tl.y;
  } else {
    expert = 0;
    m0 = mt * 256;
  }
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <int BN, int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmA2,
                     const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmOut2,
                     const GemmTcParams p) {
  using Cfg = PairCfg<BN, MODE>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* sOut = sB + STAGES * Cfg::B_BYTES;
  float* s_bias = reinterpret_cast<float*>(sOut + Cfg::STAGING);
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + Cfg::STAGING + Cfg::BIAS);  // [stage] (CTA 0's counts)
  uint64_t* empty = full + STAGES;    // [stage] ring slot free (both CTAs)
  uint64_t* tfull = empty + STAGES;   // [2] accumulator ready (both CTAs)
  uint64_t* tempty = tfull + 2;       // [2] accumulator drained (CTA 0's counts: every epilogue warp of both CTAs)
  uint64_t* stg_full = tempty + 2;    // staging tile written (epilogue warps)
  uint64_t* stg_empty = stg_full + 1;  // staging tile read by its TMA store (store thread)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stg_empty + 1);
  __shared__ int s_ntiles;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t cr = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * GEMM_EPI_WARPS);
    }
    mbar_init(stg_full, GEMM_EPI_WARPS);
    mbar_init(stg_empty, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
    if (MODE == G_MOE12) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
      tma_prefetch_desc(&tmOut2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  constexpr int KSLICE = MODE == G_FP8 ? 128 : 64;  // a K slice: one 128-byte swizzle row
  // Dense modes: the weights of this pair's first tile do not come from the
  // previous kernel (its activations do), so the first ring stages' B halves
  // go into shared memory while that kernel finishes (each stage's barrier
  // expects its A and B bytes now; A follows after the wait) and the next K
  // slices into L2 (the first 16 only: a long K, the RepEncoder's 14336,
  // streams the rest behind them, and 108 CTAs prefetching all of it would
  // flood L2).
  int pre = 0, pre_m0 = 0;
  if (!is_moe(MODE) && warp == 0 && lane == 0 && pair < p.n_tiles_dense) {
    int expert, m0, n0, mt;
    bool second;
    decode_pair_tile<BN, MODE>(p, pair, 0, expert, m0, n0, second, mt);
    pre = p.num_kb < STAGES ? p.num_kb : STAGES;
    pre_m0 = m0;
    const uint32_t full0 = mapa_shared(smem_u32(full), 0);
    constexpr uint32_t tx = 2u * uint32_t(Cfg::A_BYTES + Cfg::B_BYTES);
    for (int kb = 0; kb < pre; ++kb) {
      if (cr == 0) mbar_arrive_expect_tx(&full[kb], tx);
      tma_load_2d_pair(sB + kb * Cfg::B_BYTES, &tmB, full0 + uint32_t(kb) * 8u, kb * KSLICE, n0 + int(cr) * (BN / 2));
    }
    const int npf = p.num_kb < 16 ? p.num_kb : 16;
    for (int kb = pre; kb < npf; ++kb) tma_prefetch_2d(&tmB, kb * KSLICE, n0 + int(cr) * (BN / 2));
  }
  if (warp == 0 && lane == 0) {
    // this CTA's share of the later kernels' weights
    for (int k = 0; k < 2; ++k) {
      if (!p.pf_ptr[k]) continue;
      const size_t share = ((p.pf_bytes[k] + gridDim.x - 1) / gridDim.x + 15) & ~size_t(15);
      const size_t off = size_t(blockIdx.x) * share;
      if (off < p.pf_bytes[k]) {
        const size_t n = p.pf_bytes[k] - off < share ? p.pf_bytes[k] - off : share;
        prefetch_l2_bulk(static_cast<const char*>(p.pf_ptr[k]) + off, uint32_t(n));
      }
    }
  }
  pdl_wait();  // inputs, route tables and the error word come from earlier kernels
  pdl_trigger();  // dependents launch once this grid has passed its own wait
  // Dense modes: the A halves of the first ring stages go out now, before the
  // error word is read and the block synchronises (their operands are the
  // caller's buffers, of sizes the host checked), so that the load latency
  // overlaps that read.
  if (pre > 0) {
    const uint32_t full0 = mapa_shared(smem_u32(full), 0);
    for (int kb = 0; kb < pre; ++kb)
      tma_load_2d_pair(sA + kb * Cfg::A_BYTES, &tmA, full0 + uint32_t(kb) * 8u, kb * KSLICE, pre_m0 + 128 * int(cr));
  }
  // Expert modes: the pair's first tile entry is read together with the tile
  // count (it is used only if the tile exists)
  int2 first_tl = make_int2(0, 0);
  const int first_mt = pair / (p.N_total / BN);
  if (is_moe(MODE) && warp == 0 && lane == 0 && first_mt < p.max_mt) first_tl = p.tiles[first_mt];
  __shared__ int s_nmt;
  if (MODE == G_MOE12 && blockIdx.x == 0 && threadIdx.x == 0) {
    // the route builder's outputs are complete: the streamed combine that
    // follows may read them (and wait for this launch's second-GEMM tiles)
    st_release_gpu(const_cast<int32_t*>(p.meta) + META_MOE_GO, 1);
  }
  if (threadIdx.x == 0) {
    const int nmt = is_moe(MODE) ? p.meta[0] : 0;
    int nt = is_moe(MODE) ? nmt * (p.N_total / BN) : p.n_tiles_dense;
    if (MODE == G_MOE12) nt += nmt * (p.N2 / BN);
    s_ntiles = has_error(p.err) ? 0 : nt;
    s_nmt = nmt;
  }
  if (p.zero_ptr)
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_n; i += gridDim.x * blockDim.x)
      p.zero_ptr[i] = 0;
  __syncthreads();
  const int ntiles = s_ntiles;
  const int n_mt = s_nmt;
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // both CTAs: own halves of A and B, counted on CTA 0's full[s]
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);
      int it = pre;
      bool ok = true;
      constexpr uint32_t tx = 2u * uint32_t(Cfg::A_BYTES + Cfg::B_BYTES);
      for (int tile = pair; tile < ntiles && ok; tile += npairs) {
        int expert, m0, n0, mt;
        bool second;
        // the tile list is by M tile, the same entry for both expert GEMMs
        decode_pair_tile<BN, MODE>(p, tile, n_mt, expert, m0, n0, second, mt,
                                   tile == pair && first_mt < p.max_mt ? &first_tl : nullptr, first_mt);
        const int arow = m0 + 128 * int(cr);
        const int brow = expert * (second ? p.N2 : p.N_total) + n0 + int(cr) * (BN / 2);
        const int nkb = second ? p.N_total / 64 : p.num_kb;
        const CUtensorMap* ma = second ? &tmA2 : &tmA;
        const CUtensorMap* mb = second ? &tmB2 : &tmB;
        for (int kb = tile == pair ? pre : 0; kb < nkb; ++kb, ++it) {
          if (MODE == G_MOE12 && second && kb % (BN / 64) == 0) {
            // this K slice of the tile's A rows (H) is one first-GEMM column
            // tile of this M tile, stored by both CTAs of its pair: start on
            // it as soon as that tile is done, not the whole row
            if (!wait_flag_at_least(p.done + mt * MOE1_NT + kb / (BN / 64), 2)) {
              set_error(p.err, PTL_ERR_TIMEOUT);
              ok = false;
              break;
            }
            fence_proxy_async_global();  // the H rows were written by TMA stores
          }
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1)) {
            set_error(p.err, PTL_ERR_TIMEOUT);
            ok = false;
            break;
          }
          if (cr == 0) mbar_arrive_expect_tx(&full[s], tx);
          const uint32_t fb = full0 + uint32_t(s) * 8u;
          tma_load_2d_pair(sA + s * Cfg::A_BYTES, ma, fb, kb * KSLICE, arow);
          tma_load_2d_pair(sB + s * Cfg::B_BYTES, mb, fb, kb * KSLICE, brow);
        }
      }
      if (ntiles == 0 && cr == 0) {
        // an earlier kernel reported an error after the first stages went
        // out: let them land (both CTAs' bytes count here) before the exit
        for (int s = 0; s < pre; ++s)
          if (!mbar_wait(&full[s], 0)) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && cr == 0) {
      constexpr uint32_t idesc = MODE == G_FP8 ? umma_idesc_e4m3(256, BN) : umma_idesc_bf16(256, BN);
      int it = 0, j = 0;
      bool ok = true;
      for (int tile = pair; tile < ntiles && ok; tile += npairs, ++j) {
        int expert, m0, n0, mt;
        bool second;
        decode_pair_tile<BN, MODE>(p, tile, n_mt, expert, m0, n0, second, mt);
        const int nkb = second ? p.N_total / 64 : p.num_kb;
        const int acc = j & 1;
        if (!mbar_wait(&tempty[acc], ((j >> 1) & 1) ^ 1)) {
          set_error(p.err, PTL_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(acc * BN);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1)) {
            set_error(p.err, PTL_ERR_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * Cfg::A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * Cfg::B_BYTES);
          // four MMAs per 128-byte K slice: K = 16 bf16 or 32 e4m3 each; the
          // slices' descriptors differ by 32 bytes (+2) in the address field
          const uint64_t da = umma_desc_sw128(a0, 1024), db = umma_desc_sw128(b0, 1024);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if constexpr (MODE == G_FP8)
              umma_e4m3_ss_pair(d, da + uint64_t(2 * k), db + uint64_t(2 * k), idesc, (kb | k) != 0);
            else
              umma_bf16_ss_pair(d, da + uint64_t(2 * k), db + uint64_t(2 * k), idesc, (kb | k) != 0);
          }
          umma_commit_pair(&empty[s], 0x3);
        }
        umma_commit_pair(&tfull[acc], 0x3);
      }
    }
  } else if (warp == GEMM_STORE_WARP) {
    // Store thread (bf16 outputs): per tile, once the epilogue warps have
    // staged it, issue its TMA stores, free the staging tile as soon as the
    // stores have read it, and -- first expert GEMM -- once they are
    // complete, count the tile for the second GEMM's producers.  Its waits
    // for the stores keep the epilogue warps and the tensor core running.
    if (MODE != G_OUT && lane == 0) {
      int jj = 0;
      for (int tile = pair; tile < ntiles; tile += npairs, ++jj) {
        int expert, m0, n0, mt;
        bool second;
        decode_pair_tile<BN, MODE>(p, tile, n_mt, expert, m0, n0, second, mt);
        m0 += 128 * int(cr);
        const CUtensorMap* mo = second ? &tmOut2 : &tmOut;
        constexpr int ROUNDS = Cfg::HALF_STG ? 2 : 1;
        bool stored = true;
        for (int rd = 0; rd < ROUNDS; ++rd) {
          if (!mbar_wait(stg_full, (ROUNDS * jj + rd) & 1)) {
            set_error(p.err, PTL_ERR_TIMEOUT);
            stored = false;
            break;
          }
          if constexpr (Cfg::HALF_STG) {
            // slot s holds box 2 s + rd of the tile (64 columns each)
            tma_store_2d(mo, sOut, n0 + rd * 64, m0);
            tma_store_2d(mo, sOut + 16384, n0 + (2 + rd) * 64, m0);
          } else {
#pragma unroll 1
            for (int bx = 0; bx < BN / Cfg::BOX_COLS; ++bx)
              tma_store_2d(mo, sOut + bx * 16384, n0 + bx * Cfg::BOX_COLS, m0);
          }
          tma_store_commit();
          tma_store_wait_read();
          mbar_arrive(stg_empty);
        }
        if (!stored) break;
        if (MODE == G_MOE12) {
          // count the tile (both CTAs of the pair) once its stores are
          // complete: first-GEMM tiles for this launch's second GEMM,
          // second-GEMM tiles for the combine that follows
          tma_store_wait_all();
          fence_proxy_async_global();
          red_release_gpu_add(second ? p.done + p.max_mt * MOE1_NT + mt * MOE2_NT + n0 / BN
                                     : p.done + mt * MOE1_NT + n0 / BN,
                              1);
        }
      }
      tma_store_wait_all();
    }
  } else {
    // Epilogue warps 2..9 of each CTA: row r of this CTA's 128 rows (a warp
    // reads the TMEM lanes of its quarter, warp % 4), column half eg of the
    // tile (warps 2..5 the first half, 6..9 the second).
    const int r = 32 * (warp & 3) + lane;
    const int eg = (warp - 2) >> 2;
    const int et = int(threadIdx.x) - 64;  // 0 .. 255 over the epilogue threads
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);
    int j = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++j) {
      int expert, m0, n0, mt;
      bool second;
      decode_pair_tile<BN, MODE>(p, tile, n_mt, expert, m0, n0, second, mt);
      m0 += 128 * int(cr);  // this CTA's rows
      const int acc = j & 1;
      const int row = m0 + r;
      const float* bias_base = second ? p.bias2 : p.bias;
      const float* bb = bias_base ? bias_base + (is_moe(MODE) ? expert * (second ? p.N2 : p.N_total) : 0) + n0
                                  : nullptr;
      const bool relu = MODE == G_MOE1 || (MODE == G_MOE12 && !second);
      static_assert(BN <= 32 * 2 * GEMM_EPI_WARPS, "one bias value per epilogue thread");
      const float bv = (MODE == G_FP8 && bb && et < BN) ? __ldg(bb + et) : 0.f;
      const float swv = (MODE == G_FP8 && et < BN) ? __ldg(p.sw + n0 + et) : 0.f;
      const float sxr = (MODE == G_FP8 && row < p.M) ? __ldg(p.sx + row) : 0.f;
      constexpr int PART = Cfg::PART, NPART = BN / PART;
      constexpr int CPG = PART / 64;  // 32-column chunks of a part per column half
      static_assert(PART % 64 == 0, "a part splits into two halves of whole chunks");
      constexpr int NRES = MODE == G_OUT ? PART / 16 : 1;
      uint4 res[NRES];  // this thread's half of its residual row, one part at a time
      auto load_res = [&](int pt) {
        if (MODE == G_OUT) {
          const uint4* src = reinterpret_cast<const uint4*>(p.resid + size_t(row < p.M ? row : 0) * D + n0 + pt * PART +
                                                            eg * (PART / 2));
#pragma unroll
          for (int q = 0; q < NRES; ++q) res[q] = row < p.M ? __ldg(src + q) : make_uint4(0, 0, 0, 0);
        }
      };
      load_res(0);
      const bool leader = warp == 2 && lane == 0;
      // the fp32 output stages in parts through the leader's own stores; the
      // bf16 outputs go through the store thread
      // this tile's bias (+ scales) in buffer j % 2: the barrier below is
      // passed only once every thread has finished tile j - 1, which read
      // the other buffer
      float* const sb = s_bias + (j & 1) * (Cfg::BIAS / 8);
      if (MODE == G_FP8 && et < BN) {
        sb[et] = bv;
        sb[BN + et] = swv;
      }
      if (MODE == G_FP8) named_barrier(1, 32 * GEMM_EPI_WARPS);
      if (!mbar_wait(&tfull[acc], (j >> 1) & 1)) {
        set_error(p.err, PTL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + uint32_t(acc * BN) + lane_off;
      // bias (+ FP8 scales, + ReLU) on 32 accumulator columns starting at `col`
      auto finish32 = [&](float (&v)[32], int col) {
        if (MODE == G_FP8) {  // code products times the row's and the column's scales
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 s4 = *reinterpret_cast<const float4*>(sb + BN + col + 4 * q);
            v[4 * q] = v[4 * q] * sxr * s4.x;
            v[4 * q + 1] = v[4 * q + 1] * sxr * s4.y;
            v[4 * q + 2] = v[4 * q + 2] * sxr * s4.z;
            v[4 * q + 3] = v[4 * q + 3] * sxr * s4.w;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          // the bias of 32 columns: the same addresses for the whole warp
          // (16-byte aligned: the entry points check the bias pointers)
          const float4 b4 = MODE == G_FP8 ? *reinterpret_cast<const float4*>(sb + col + 4 * q)
                            : bb          ? __ldg(reinterpret_cast<const float4*>(bb + col + 4 * q))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
          v[4 * q] += b4.x;
          v[4 * q + 1] += b4.y;
          v[4 * q + 2] += b4.z;
          v[4 * q + 3] += b4.w;
        }
        if (relu) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i], 0.f);
        }
      };
      if constexpr (MODE != G_OUT) {
        // bf16 output, staged in one round (the whole tile) or two of 128
        // columns (a box from each column half; column half eg writes slot
        // eg).  A round's columns go through registers first; after the last
        // round's TMEM reads the accumulator is released (the tensor core can
        // start the tile after next) before the staging tile is waited for.
        constexpr int ROUNDS = Cfg::HALF_STG ? 2 : 1, CPR = CPG / ROUNDS;
        static_assert(!Cfg::HALF_STG || CPG == 4, "half staging: two boxes per column half");
        bool staged = true;
#pragma unroll
        for (int rd = 0; rd < ROUNDS; ++rd) {
          uint32_t pk[CPR][16];
#pragma unroll
          for (int k = 0; k < CPR; ++k) {
            const int col = 32 * (eg * CPG + rd * CPR + k);  // column within the tile
            uint32_t raw[32];
            tmem_ld32(taddr + col, raw);
            tmem_ld_wait_regs(raw);
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
            finish32(v, col);
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[k][i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          }
          if (rd == ROUNDS - 1) {
            // this warp's rows of the accumulator are read: release it on CTA 0
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0 + uint32_t(acc) * 8u);
          }
          // the previous round's stores have read the staging tile
          const int R = ROUNDS * j + rd;
          if (R > 0 && !mbar_wait(stg_empty, (R - 1) & 1)) {
            set_error(p.err, PTL_ERR_TIMEOUT);
            staged = false;
            break;
          }
#pragma unroll
          for (int k = 0; k < CPR; ++k) {
            // 32 bf16 = half a box row: 16-byte chunks (c%2)*4 .. +3 of box
            // c/2 (whole tile) or of slot eg (half staging)
            const int c = eg * CPG + rd * CPR + k;
            const int box = Cfg::HALF_STG ? eg : (c >> 1);
            const uint32_t rowa = smem_u32(sOut + box * 16384) + r * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int chunk = (c & 1) * 4 + q;
              st_shared_v4(rowa + ((chunk ^ (r & 7)) << 4), pk[k][4 * q], pk[k][4 * q + 1], pk[k][4 * q + 2],
                           pk[k][4 * q + 3]);
            }
          }
          // staged: hand the round to the store thread (one arrival per warp)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(stg_full);
        }
        if (!staged) break;
      } else {
#pragma unroll 1
        for (int pt = 0; pt < NPART; ++pt) {
          // buffer pt % 2 was last staged two parts ago (in this tile or the
          // previous one): its store must have read it; the previous part's
          // store may still be running
          if (pt > 0) load_res(pt);
          if (leader) tma_store_wait_read_but_one();
          named_barrier(1, 32 * GEMM_EPI_WARPS);
          uint8_t* const buf = sOut + (pt & 1) * (Cfg::STAGING / 2);
#pragma unroll
          for (int cc = 0; cc < CPG; ++cc) {
            const int c = eg * CPG + cc;  // chunk within the part
            const int col = pt * PART + 32 * c;  // column within the tile
            uint32_t raw[32];
            tmem_ld32(taddr + col, raw);
            tmem_ld_wait_regs(raw);
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
            finish32(v, col);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 u = res[4 * cc + q];
              const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h2[i]);
                v[8 * q + 2 * i] += f.x;
                v[8 * q + 2 * i + 1] += f.y;
              }
            }
            // 32 fp32 = one 128-byte box row: box c of the part, chunks 0..7
            const uint32_t rowa = smem_u32(buf + c * 16384) + r * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_shared_v4(rowa + ((q ^ (r & 7)) << 4), __float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                           __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
          }
          if (pt == NPART - 1) {
            // this warp's rows of the accumulator are read: release it on CTA 0
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0 + uint32_t(acc) * 8u);
          }
          fence_proxy_async_smem();
          named_barrier(1, 32 * GEMM_EPI_WARPS);
          if (leader) {
            const CUtensorMap* mo = second ? &tmOut2 : &tmOut;
#pragma unroll 1
            for (int bx = 0; bx < PART / Cfg::BOX_COLS; ++bx)
              tma_store_2d(mo, buf + bx * 16384, n0 + pt * PART + bx * Cfg::BOX_COLS, m0);
            tma_store_commit();
          }
        }
      }
    }
    if (MODE == G_OUT && warp == 2 && lane == 0) tma_store_wait_all();
  }
  __syncwarp();  // the single-lane roles rejoin their warps before the cluster barrier
  tc_fence_before();
  cluster_sync();  // no MMA, TMEM read or remote arrival of either CTA is outstanding
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host

// Launches the CTA-pair kernel: clusters of two CTAs, one pair per two SMs.
template <int BN, int MODE>
static int launch_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& out,
                       const GemmTcParams& p, int tiles_bound, cudaStream_t st, const CUtensorMap* a2 = nullptr,
                       const CUtensorMap* b2 = nullptr, const CUtensorMap* out2 = nullptr) {
  // co-resident clusters of two (one CTA per SM) on the current device,
  // found once per device together with the kernel's shared-memory limit
  static PerDevice max_pairs_dev;
  const int smem = PairCfg<BN, MODE>::SMEM;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const int max_pairs = max_pairs_dev.get([&] {
    if (cudaFuncSetAttribute(gemm_pair_kernel<BN, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return -1;
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<BN, MODE>, &q) != cudaSuccess || n < 1)
      n = num_sms() / 2;
    return n;
  });
  if (max_pairs < 1) return -1;
  int pairs = max_pairs;
  if (tiles_bound < pairs) pairs = tiles_bound;
  if (pairs < 1) pairs = 1;
  cfg.gridDim = dim3(2 * pairs);
  if (cudaLaunchKernelEx(&cfg, gemm_pair_kernel<BN, MODE>, a, b, out, a2 ? *a2 : a, b2 ? *b2 : b,
                         out2 ? *out2 : out, p) != cudaSuccess)
    return -1;
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -1;
}

int launch_gemm_qkv(const CUtensorMap& xn, const CUtensorMap& w, const CUtensorMap& qkv_out,
                    const float* bias, void* qkv, int T, int32_t* err, cudaStream_t st, const void* pf0,
                    size_t pf0_bytes, const void* pf1, size_t pf1_bytes) {
  GemmTcParams p{};
  p.pf_ptr[0] = pf0;
  p.pf_bytes[0] = pf0_bytes;
  p.pf_ptr[1] = pf1;
  p.pf_bytes[1] = pf1_bytes;
  p.M = T;
  p.N_total = QKV_N;
  p.num_kb = D / 64;
  p.n_tiles_dense = ((T + 255) / 256) * (QKV_N / QKV_BN);  // 256-row pair tiles
  p.bias = bias;
  p.out = static_cast<__nv_bfloat16*>(qkv);
  p.ldo = QKV_N;
  p.err = err;
  return launch_pair<QKV_BN, G_QKV>(xn, w, qkv_out, p, p.n_tiles_dense, st);
}

int launch_gemm_rep(const CUtensorMap& normed, const CUtensorMap& w, const CUtensorMap& out_map,
                    const float* bias, int T, int32_t* err, cudaStream_t st) {
  GemmTcParams p{};
  p.M = T;
  p.N_total = D;
  p.num_kb = REP_W / 64;
  p.n_tiles_dense = ((T + 255) / 256) * (D / 256);  // 256-row pair tiles
  p.bias = bias;
  p.ldo = D;
  p.err = err;
  return launch_pair<256, G_QKV>(normed, w, out_map, p, p.n_tiles_dense, st);
}

int launch_gemm_out(const CUtensorMap& attn, const CUtensorMap& w, const CUtensorMap& x1_out,
                    const float* bias, const void* x, void* x1, int T, int32_t* err, cudaStream_t st) {
  GemmTcParams p{};
  p.M = T;
  p.N_total = D;
  p.num_kb = D / 64;
  p.n_tiles_dense = ((T + 255) / 256) * (D / OUT_BN);  // 256-row pair tiles
  p.bias = bias;
  p.resid = static_cast<const __nv_bfloat16*>(x);
  p.out_f32 = static_cast<float*>(x1);
  p.ldo = D;
  p.err = err;
  return launch_pair<OUT_BN, G_OUT>(attn, w, x1_out, p, p.n_tiles_dense, st);
}

int launch_gemm_fp8(const CUtensorMap& xq, const CUtensorMap& wq, const CUtensorMap& out_map, const float* sx,
                    const float* sw, const float* bias, int M, int N, int Kd, int32_t* err, cudaStream_t st) {
  GemmTcParams p{};
  p.M = M;
  p.N_total = N;
  p.num_kb = Kd / 128;  // 128 e4m3 per 128-byte swizzle row
  p.n_tiles_dense = ((M + 255) / 256) * (N / 256);
  p.bias = bias;
  p.ldo = N;
  p.err = err;
  p.sx = sx;
  p.sw = sw;
  return launch_pair<256, G_FP8>(xq, wq, out_map, p, p.n_tiles_dense, st);
}

int launch_gemm_moe1(const CUtensorMap& xperm, const CUtensorMap& w1, const CUtensorMap& hbuf_out,
                     const float* b1, const WsLayout& L, char* ws, cudaStream_t st) {
  GemmTcParams p{};
  p.N_total = F;
  p.num_kb = D / 64;
  p.bias = b1;
  p.out = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
  p.ldo = F;
  p.tiles = reinterpret_cast<const int2*>(ws + L.tiles);
  p.meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
  p.max_mt = int(L.max_tiles);
  p.err = reinterpret_cast<int32_t*>(ws + L.err);
  // the routing state of this layer (per-chunk expert counts, look-back
  // state, contiguous in the workspace) is consumed: clear it for the next
  // layer's gate
  p.zero_ptr = reinterpret_cast<int32_t*>(ws + L.chunk_cnt);
  p.zero_n = int((L.clear_end - L.chunk_cnt) / 4);
  return launch_pair<MOE1_BN, G_MOE1>(xperm, w1, hbuf_out, p, int(L.max_tiles) * (F / MOE1_BN), st);
}

int launch_gemm_moe12(const CUtensorMap& xperm, const CUtensorMap& w1, const CUtensorMap& hbuf,
                      const CUtensorMap& w2, const CUtensorMap& ybuf_out, const float* b1, const float* b2,
                      const WsLayout& L, char* ws, cudaStream_t st) {
  static_assert(MOE1_BN == GEMM2_BN, "both expert GEMMs share one tile shape");
  GemmTcParams p{};
  p.N_total = F;
  p.num_kb = D / 64;
  p.bias = b1;
  p.N2 = D;
  p.bias2 = b2;
  p.tiles = reinterpret_cast<const int2*>(ws + L.tiles);
  p.meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
  p.max_mt = int(L.max_tiles);
  p.err = reinterpret_cast<int32_t*>(ws + L.err);
  p.done = reinterpret_cast<int32_t*>(ws + L.moe_done);
  // the routing state of this layer is consumed: clear it for the next layer
  p.zero_ptr = reinterpret_cast<int32_t*>(ws + L.chunk_cnt);
  p.zero_n = int((L.lb - L.chunk_cnt) / 4 + 32 + 32 * L.n_gchunks);
  return launch_pair<MOE1_BN, G_MOE12>(xperm, w1, hbuf, p, int(L.max_tiles) * (F + D) / MOE1_BN, st, &hbuf, &w2,
                                       &ybuf_out);
}

int launch_gemm_moe2(const CUtensorMap& hbuf, const CUtensorMap& w2, const CUtensorMap& ybuf_out,
                     const float* b2, const WsLayout& L, char* ws, cudaStream_t st) {
  GemmTcParams p{};
  p.N_total = D;
  p.num_kb = F / 64;
  p.bias = b2;
  p.out = reinterpret_cast<__nv_bfloat16*>(ws + L.ybuf);
  p.ldo = D;
  p.tiles = reinterpret_cast<const int2*>(ws + L.tiles);
  p.meta = reinterpret_cast<const int32_t*>(ws + L.route_meta);
  p.max_mt = int(L.max_tiles);
  p.err = reinterpret_cast<int32_t*>(ws + L.err);
  return launch_pair<GEMM2_BN, G_MOE2>(hbuf, w2, ybuf_out, p, int(L.max_tiles) * (D / GEMM2_BN), st);
}

}  // namespace ptl
