// The two projections around the attention of a C2PSA-style block, as
// tcgen05 GEMMs whose data movement is fused with the attention layout:
//
//   qkv:  [q | k | v] = x W_qkv^T + b_qkv,  x [B, N, C], W_qkv [3 C, C]
//         (the qkv Linear of the YOLO11 x FlashAttention-2 page (kwkr.cn),
//         section 2.2, whose output is reshaped to [B, N, 3, H, d] and
//         permuted to three [B, H, N, d] tensors).  The epilogue writes each
//         output column straight to its place in q, k or v [B, H, N, d], so
//         no reshape / permute / contiguous pass follows.
//   proj: y = o' W_o^T + b_o,  o' the [B, N, H d] view of the attention
//         output o [B, H, N, d] (the proj Linear of the same section, after
//         the transpose back).  The A operand is loaded from o itself through
//         a 4-D tensor map (d, N, H, B), so the transpose is never
//         materialised.
//
// "FlashAttention 深度解读" (coreui.cn), section "实现 2", fuses QKV
// generation with the attention; here the fusion is of the layout changes
// into the producing and consuming GEMMs, which is where the extra HBM
// round trips of the unfused block are.
//
// One CTA per 128 x 128 output tile; K in 64-wide steps through a 2-stage
// TMA ring (128-byte swizzle, both operands K-major, the layout and
// descriptors of the attention kernel's S = Q K^T); warp 4 loads, warp 5
// issues tcgen05.mma (fp32 accumulator in TMEM), warps 0-3 read the
// accumulator back (one row per thread), add the bias and store.  With K as
// short as the block's channel count (256 .. 1024) a tile is mostly load
// latency and epilogue, so the ring is kept small enough (65 KB) for three
// CTAs per SM: one CTA's epilogue and start-up overlap the others' loads and
// MMAs (4 stages and one CTA per SM took 35-50 % longer).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "attn_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int PROJ_THREADS = 192;
constexpr int PROJ_STAGES = 2;
constexpr int PROJ_CTAS_PER_SM = 3;  // shared memory 3 x 65 KB, TMEM 3 x 128 columns
constexpr int PROJ_LOAD_WARP = 4;
constexpr int PROJ_MMA_WARP = 5;

enum ProjMode : int {
  PROJ_QKV = 0,  // A = x [M = B N, K = C] (2-D map), epilogue scatters into q, k, v
  PROJ_OUT = 1,  // A = o [B, H, N, d] read as [B N, H d] (4-D map), row-major epilogue
};

struct ProjParams {
  const float* bias;  // [N_out] fp32, or nullptr
  void* out0;         // PROJ_QKV: q; PROJ_OUT: y [B, N, N_out]
  void* out1;         // PROJ_QKV: k
  void* out2;         // PROJ_QKV: v
  int B, N, K, N_out;
  int H, d;           // heads and head dim (PROJ_QKV: of q, k, v; PROJ_OUT: of o)
  int m_tiles;        // PROJ_QKV: ceil(B N / 128); PROJ_OUT: ceil(N / 128) per batch
};

struct ProjSmem {
  static constexpr int SLAB = 128 * 64 * 2;  // 128 rows x 64 16-bit columns
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + PROJ_STAGES * SLAB;
  static constexpr int BAR_OFF = B_OFF + PROJ_STAGES * SLAB;
  static constexpr int FULL = 0, EMPTY = PROJ_STAGES, ACC = 2 * PROJ_STAGES;
  static constexpr int NUM_BARS = ACC + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int BYTES = MISC_OFF + 16 + 1024;
};

template <bool BF16, int MODE>
__global__ void __launch_bounds__(PROJ_THREADS, PROJ_CTAS_PER_SM)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const ProjParams p) {
  using L = ProjSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + L::BAR_OFF + 8u * i; };
  const int n_tile = blockIdx.x;
  const int m_tile = blockIdx.y;
  const int k_steps = p.K / 64;
  // PROJ_OUT: this tile is rows n0 .. n0 + 127 of batch b
  const int b_out = MODE == PROJ_OUT ? m_tile / p.m_tiles : 0;
  const int n0_out = MODE == PROJ_OUT ? (m_tile - b_out * p.m_tiles) * 128 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PROJ_STAGES; ++s) {
      mbar_init(bar(L::FULL + s), 1);
      mbar_init(bar(L::EMPTY + s), 1);
    }
    mbar_init(bar(L::ACC), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == PROJ_LOAD_WARP && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == PROJ_MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == PROJ_LOAD_WARP) {
    const bool leader = elect_one();
    int ks = 0;
    for (; ks < k_steps; ++ks) {
      const int s = ks % PROJ_STAGES;
      if (ks >= PROJ_STAGES &&
          !__all_sync(0xffffffffu, wait_phase(bar(L::EMPTY + s), (ks / PROJ_STAGES - 1) & 1,
                                              abort_flag, SITE_LOAD_KV_EMPTY)))
        break;
      if (leader) {
        mbar_arrive_expect_tx(bar(L::FULL + s), 2 * L::SLAB);
        const int k0 = ks * 64;
        if constexpr (MODE == PROJ_QKV) {
          tma_load_3d(sbase + L::A_OFF + s * L::SLAB, &tm_a, bar(L::FULL + s), k0, m_tile * 128, 0);
        } else {
          tma_load_4d(sbase + L::A_OFF + s * L::SLAB, &tm_a, bar(L::FULL + s), k0 % p.d, n0_out,
                      k0 / p.d, b_out);
        }
        tma_load_3d(sbase + L::B_OFF + s * L::SLAB, &tm_b, bar(L::FULL + s), k0, n_tile * 128, 0);
      }
      __syncwarp();
    }
    for (int m = ks > PROJ_STAGES ? ks - PROJ_STAGES : 0; m < ks; ++m)
      wait_phase(bar(L::FULL + m % PROJ_STAGES), (m / PROJ_STAGES) & 1, abort_flag, SITE_DRAIN,
                 false);
    __syncwarp();
  } else if (warp == PROJ_MMA_WARP) {
    const bool leader = elect_one();
    constexpr uint32_t IDESC = idesc_f16(BF16, false, false, 128, 128);
    const uint64_t a_desc = sw128_desc(sbase + L::A_OFF, 16, 1024);
    const uint64_t b_desc = sw128_desc(sbase + L::B_OFF, 16, 1024);
    for (int ks = 0; ks < k_steps; ++ks) {
      const int s = ks % PROJ_STAGES;
      if (!__all_sync(0xffffffffu, wait_phase(bar(L::FULL + s), (ks / PROJ_STAGES) & 1, abort_flag,
                                              SITE_MMA_KV_FULL)))
        break;
      tc_fence_after();
      if (leader) {
        const uint32_t so = s * (L::SLAB >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem_base, a_desc + so + kk * 2, b_desc + so + kk * 2, IDESC,
                 (ks > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(L::EMPTY + s));
      }
      __syncwarp();
    }
    if (leader) mma_commit(bar(L::ACC));
    __syncwarp();
    wait_phase(bar(L::ACC), 0, abort_flag, SITE_DRAIN, false);
    __syncwarp();
  } else {
    // epilogue: thread = output row r of the tile
    const int r = warp * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    const bool ok = __all_sync(0xffffffffu, wait_phase(bar(L::ACC), 0, abort_flag,
                                                       SITE_SOFTMAX_O_READY));
    if (ok && k_steps > 0) {
      tc_fence_after();
      long long row;  // PROJ_QKV: row of x (b N + n); PROJ_OUT: n within batch b_out
      bool row_ok;
      long long qkv_b = 0, qkv_n = 0;  // PROJ_QKV: the row's batch and position, split once
      if constexpr (MODE == PROJ_QKV) {
        row = static_cast<long long>(m_tile) * 128 + r;
        row_ok = row < static_cast<long long>(p.B) * p.N;
        qkv_b = row / p.N;
        qkv_n = row - qkv_b * p.N;
      } else {
        row = n0_out + r;
        row_ok = row < p.N;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t a[32];
        tmem_ld32(t_row + c0, a);
        tmem_wait_ld_regs(a);
        const int col0 = n_tile * 128 + c0;  // first output column of this chunk
        if (!row_ok || col0 >= p.N_out) continue;
        float v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float bias = (p.bias != nullptr && col0 + c < p.N_out) ? p.bias[col0 + c] : 0.f;
          v[c] = __uint_as_float(a[c]) + bias;
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack2<BF16>(v[2 * c], v[2 * c + 1]);
        uint16_t* dst;
        if constexpr (MODE == PROJ_QKV) {
          // column c of [q | k | v]: tensor c / C, head (c % C) / d, element c % d; a
          // 32-column chunk never straddles a head (d is 64 or 128)
          const int C = p.H * p.d;
          const int which = col0 / C, rem = col0 - which * C;
          const int h = rem / p.d, dd = rem - h * p.d;
          const long long b = qkv_b, n = qkv_n;
          void* base = which == 0 ? p.out0 : (which == 1 ? p.out1 : p.out2);
          dst = static_cast<uint16_t*>(base) + ((b * p.H + h) * p.N + n) * p.d + dd;
        } else {
          dst = static_cast<uint16_t*>(p.out0) +
                (static_cast<long long>(b_out) * p.N + row) * p.N_out + col0;
        }
        if (col0 + 32 <= p.N_out) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            reinterpret_cast<uint4*>(dst)[v4] =
                make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (col0 + c < p.N_out)
              dst[c] = static_cast<uint16_t>((c & 1) ? (pk[c / 2] >> 16) : (pk[c / 2] & 0xFFFFu));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == PROJ_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 128);
  }
}

}  // namespace attn_sm100
