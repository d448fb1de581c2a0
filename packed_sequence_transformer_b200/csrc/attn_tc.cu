// attn_tc.cu -- jagged block-diagonal causal attention on tcgen05.
//
// Work item = (user u, query block b, head h): 128 query rows of one user.
// The items are listed on the device from cu_seqlens, heaviest first (a
// block b needs b + 1 key blocks: the key loop stops at the diagonal block,
// so no [S,S] mask and no block above the diagonal is ever touched).
//
// Per item (4 warps, thread i <-> query row i <-> TMEM lane i):
//   TMA: Q tile [128 x 64] once, then per key block K and V tiles [128 x 64]
//        straight out of the packed qkv rows (128-byte swizzle);
//   S = Q K^T    tcgen05.mma M=128 N=128 K=16 x4 into TMEM columns [0,128);
//   softmax      each thread reads its S row from TMEM, masks keys beyond
//                its own position (and beyond the user), keeps the running
//                max m and sum l in fp32 (base-2 exponent, scale folded in),
//                and writes P = exp2(s - m) in bf16 into shared memory in the
//                K-major swizzled layout the tensor core reads;
//   PV = P V     tcgen05.mma M=128 N=64 K=16 x8 (V is the MN-major operand)
//                into TMEM columns [128,192); the thread folds it into its
//                fp32 output row, O = O * exp2(m_old - m_new) + PV.
// Finally O / l is written as bf16 for the rows that belong to the user.
// Tiles that run past the user (into the next user or past T) are masked;
// TMA zero-fills rows past T.  All waits are bounded.
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
constexpr int ATT_SMEM = 5 * ATT_TILE_BYTES + 1024 + 128;

__global__ void __launch_bounds__(128, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const int32_t* __restrict__ cu,
                   const int2* __restrict__ items, const int32_t* __restrict__ item_count,
                   __nv_bfloat16* __restrict__ out, int32_t* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + ATT_TILE_BYTES;
  uint8_t* sV = smem + 2 * ATT_TILE_BYTES;
  uint8_t* sP = smem + 3 * ATT_TILE_BYTES;  // two 64-key column blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 5 * ATT_TILE_BYTES);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_kv = bars + 1;
  uint64_t* bar_s = bars + 2;
  uint64_t* bar_o = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  __shared__ int s_skip;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int item = blockIdx.x / H, h = blockIdx.x % H;
  pdl_trigger();
  pdl_wait();  // qkv, the work list and the error word come from earlier kernels
  if (tid == 0) {
    const int skip = (has_error(err) || item >= *item_count) ? 1 : 0;
    s_skip = skip;
    if (!skip) {
      mbar_init(bar_q, 1);
      mbar_init(bar_kv, 1);
      mbar_init(bar_s, 1);
      mbar_init(bar_o, 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  if (s_skip) return;
  const int2 it = items[item];
  const int s0 = cu[it.x];
  const int L = cu[it.x + 1] - s0;
  const int qb = it.y;
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + 128;
  const uint32_t lane_off = uint32_t(32 * warp) << 16;

  const int qi = qb * ATT_BLK + tid;      // query position inside the user
  const int qlim = min(qi, L - 1);        // keys 0..qlim are visible
  const float c2 = 0.125f * 1.4426950408889634f;  // softmax scale * log2(e)
  constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128);
  constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 64, 0, 1);

  if (tid == 0) {
    tma_prefetch_desc(&tm_qkv);
    mbar_arrive_expect_tx(bar_q, ATT_TILE_BYTES);
    tma_load_2d(sQ, &tm_qkv, bar_q, h * DH, s0 + qb * ATT_BLK);
  }
  float o[DH];
#pragma unroll
  for (int d = 0; d < DH; ++d) o[d] = 0.f;
  float m = -INFINITY, l = 0.f;
  bool ok = true;

  for (int kb = 0; kb <= qb && ok; ++kb) {
    const uint32_t ph = kb & 1;
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_kv, 2 * ATT_TILE_BYTES);
      tma_load_2d(sK, &tm_qkv, bar_kv, D + h * DH, s0 + kb * ATT_BLK);
      tma_load_2d(sV, &tm_qkv, bar_kv, 2 * D + h * DH, s0 + kb * ATT_BLK);
      if (mbar_wait(bar_q, 0) && mbar_wait(bar_kv, ph)) {
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ss(tS, umma_desc_sw128(q0 + 32 * k, 1024), umma_desc_sw128(k0 + 32 * k, 1024),
                       idesc_qk, k != 0);
        umma_commit(bar_s);
      } else {
        set_error(err, PTL_ERR_TIMEOUT);
      }
    }
    if (!mbar_wait(bar_s, ph)) {
      set_error(err, PTL_ERR_TIMEOUT);
      ok = false;
    }
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();

    // pass 1: row maximum over the visible keys of this block
    const int kbase = kb * ATT_BLK;
    float mx = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t raw[32];
      tmem_ld32(tS + lane_off + 32 * c, raw);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (kbase + 32 * c + i <= qlim) mx = fmaxf(mx, __uint_as_float(raw[i]));
    }
    const float m_new = fmaxf(m, mx * c2);
    const float alpha = exp2f(m - m_new);
    // pass 2: probabilities -> bf16 P in shared memory (K-major, swizzled)
    float lsum = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t raw[32];
      tmem_ld32(tS + lane_off + 32 * c, raw);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const int j = kbase + 32 * c + i;
        const float p0 = (j <= qlim) ? exp2f(__uint_as_float(raw[i]) * c2 - m_new) : 0.f;
        const float p1 = (j + 1 <= qlim) ? exp2f(__uint_as_float(raw[i + 1]) * c2 - m_new) : 0.f;
        lsum += p0 + p1;
        pk[i >> 1] = pack_bf16x2(p0, p1);
      }
      // keys 32c..32c+31 live in column block c/2, 16-byte chunks (c%2)*4 .. +3
      const uint32_t row_addr = smem_u32(sP + (c >> 1) * ATT_TILE_BYTES) + tid * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int chunk = (c & 1) * 4 + q;
        st_shared_v4(row_addr + ((chunk ^ (tid & 7)) << 4), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                     pk[4 * q + 3]);
      }
    }
    l = l * alpha + lsum;
    m = m_new;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t p0 = smem_u32(sP), v0 = smem_u32(sV);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        umma_bf16_ss(tO, umma_desc_sw128(p0 + (k >> 2) * ATT_TILE_BYTES + 32 * (k & 3), 1024),
                     umma_desc_sw128(v0 + k * 2048, 1024, 8192), idesc_pv, k != 0);
      umma_commit(bar_o);
    }
    if (!mbar_wait(bar_o, ph)) {
      set_error(err, PTL_ERR_TIMEOUT);
      ok = false;
    }
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t raw[32];
      tmem_ld32(tO + lane_off + 32 * c, raw);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) o[32 * c + i] = o[32 * c + i] * alpha + __uint_as_float(raw[i]);
    }
    tc_fence_before();
    __syncthreads();
  }

  if (ok && qi < L) {
    const float inv = 1.0f / l;
    uint4* dst = reinterpret_cast<uint4*>(out + size_t(s0 + qi) * D + h * DH);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint4 u;
      u.x = pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
      u.y = pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
      u.z = pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
      u.w = pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
      dst[q] = u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

int launch_attn_tc(const CUtensorMap& qkv_map, void* out, const int32_t* cu, const WsLayout& L,
                   char* ws, cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_SMEM) !=
        cudaSuccess)
      return -1;
    configured = true;
  }
  if (launch_k(attn_tc_kernel, dim3(unsigned(L.max_items * H)), dim3(128), ATT_SMEM, st, qkv_map, cu,
               reinterpret_cast<const int2*>(ws + L.items), reinterpret_cast<const int32_t*>(ws + L.item_count),
               static_cast<__nv_bfloat16*>(out), reinterpret_cast<int32_t*>(ws + L.err)) != 0)
    return -1;
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace ptl
