// Exact attention backward for sm_100a (B200): the gradients dQ, dK, dV of
//   O = softmax(Q K^T * scale [+ top-left causal mask]) V
// for an output gradient dO, with the softmax recomputed from the forward's
// saved logsumexp instead of being stored ("YOLOv12推理速度翻倍秘诀：Flash
// Attention加持" (0539edu.com), section 1: recompute the softmax
// intermediates in the backward pass; YOLO11 x FlashAttention-2 (kwkr.cn),
// sections 2.3 and 4.3: the statistics kept for the backward).  For one
// (batch, head), with P = exp(S - lse):
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three kernels:
//   * bwd_prep_kernel: D_i = sum_c dO_ic O_ic and lse_i * log2 e, both padded
//     to whole 128-row tiles (pad rows get D = 0 and +inf, so their P is 0),
//     and zeroes the fp32 dQ accumulator;
//   * bwd_main_kernel: one CTA per (128-key tile, batch-head).  K_j and V_j
//     stay in shared memory; for every query tile i that sees key tile j the
//     tensor core computes S^T = K_j Q_i^T and dP^T = V_j dO_i^T into tensor
//     memory (one TMEM lane per key), two softmax warpgroups turn them into
//     P^T (written back over S^T as 16-bit pairs) and dS^T (written to a
//     128-byte-swizzled shared-memory tile), and the tensor core accumulates
//     dV += P^T dO_i and dK += dS^T Q_i in TMEM and computes dQ_ij = dS K_j,
//     which a readout warpgroup stages in shared memory and adds into the
//     fp32 dQ accumulator with TMA bulk reductions;
//   * bwd_dq_kernel: dQ = scale * accumulator, rounded to the input dtype.
//
// Every operand layout is one the forward already uses: K-major tiles as the
// first and second operands of S^T and dP^T, MN-major tiles (head dim
// contiguous) as the second operand of dV, dK and dQ, and the MN-major view
// of the dS^T tile (queries contiguous) as the first operand of dQ.
// Every wait is bounded like the forward's (status word, abort flag).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "attn_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int BWD_THREADS = 448;   // 14 warps
constexpr int BWD_LOAD_WARP = 12;  // TMA loads of K, V, Q_i, dO_i
constexpr int BWD_MMA_WARP = 13;   // issues every tcgen05.mma
// warps 0-3 / 4-7: softmax warpgroups, query columns 0-63 / 64-127 of a tile;
// warps 8-11: dQ readout warpgroup

struct BwdParams {
  void* dk;               // [B, H, Nk, D]
  void* dv;               // [B, H, Nk, D]
  float* dq_acc;          // [B, H, Nq, D] fp32, zeroed by the prep kernel
  const float* lse2;      // [B, H, Nq_pad]: lse * log2 e, +inf on pad rows
  const float* dsum;      // [B, H, Nq_pad]: D = rowsum(dO * O), 0 on pad rows
  int Nq, Nk, BH;
  int nq_tiles, nk_tiles, nq_pad;
  int causal;
  float scale;            // applied to dK here and to dQ in bwd_dq_kernel
  float scale_log2;       // scale * log2 e
};

template <int D>
struct BwdSmem {
  static constexpr int HALF_BYTES = 128 * 64 * 2;  // one 64-column, 128-byte-swizzled slab
  static constexpr int TILE_BYTES = (D / 64) * HALF_BYTES;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE_BYTES;
  static constexpr int RING_OFF = V_OFF + TILE_BYTES;  // + stage * 2 tiles: Q_i, then dO_i
  static constexpr int STAGES = 2;
  static constexpr int DS_OFF = RING_OFF + STAGES * 2 * TILE_BYTES;  // dS^T, 2 slabs of 64 queries
  static constexpr int DS_BYTES = 2 * HALF_BYTES;
  // At d = 64 each stage also holds the tile's 128 lse (base 2) and D values,
  // copied in with Q_i and dO_i; d = 128 has no room and reads them from
  // global memory.
  static constexpr bool STATS_IN_SMEM = (D == 64);
  static constexpr int STATS_OFF = DS_OFF + DS_BYTES;  // + stage * 1024: lse2[128], then D[128]
  // The readout adds each dQ_ij tile (128 rows x D fp32, 32-column boxes with
  // the 128-byte swizzle) to the accumulator with TMA bulk reductions from
  // shared memory.  At d = 64 it stages the tile in one of two 32 KB slots of
  // its own; at d = 128, which has no room for them, in the ring stage of the
  // tile itself (Q_i and dO_i take exactly 64 KB, and every MMA that read them
  // is done when dQ_ij is), and the readout, not the MMA warp, then hands the
  // stage back to the loader once the reductions have read it.
  static constexpr bool DQ_IN_STAGE = (D == 128);
  static constexpr int DQ_OFF = STATS_OFF + (STATS_IN_SMEM ? STAGES * 1024 : 0);  // + slot * 32 KB
  static constexpr int BAR_OFF = DQ_OFF + (DQ_IN_STAGE ? 0 : 2 * 32768);
  // mbarriers
  static constexpr int KV_FULL = 0;
  static constexpr int RING_FULL = 1;                // + stage
  static constexpr int RING_EMPTY = RING_FULL + STAGES;  // + stage
  static constexpr int S_READY = RING_EMPTY + STAGES;
  static constexpr int DP_READY = S_READY + 1;
  static constexpr int P_READY = DP_READY + 1;    // 256 softmax threads arrive
  static constexpr int DS_READY = P_READY + 1;    // 256 softmax threads arrive
  static constexpr int DQ_READY = DS_READY + 1;   // dK and dQ of the tile done
  static constexpr int DQ_FREE = DQ_READY + 1;    // 128 readout threads arrive
  static constexpr int DONE = DQ_FREE + 1;        // every MMA done
  static constexpr int RO_SYNC = DONE + 1;        // rendezvous of the 128 readout threads
  static constexpr int NUM_BARS = RO_SYNC + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;  // TMEM address, abort flag
  static constexpr int BYTES = MISC_OFF + 16 + 1024;      // + slack to align the base to 1 KB
  static_assert(BYTES <= 232448, "shared memory budget");
  // TMEM columns (512 allocated)
  // S^T fp32 [key][query]; P^T as 16-bit pairs, queries 64 w .. 64 w + 63 in
  // columns 64 w .. 64 w + 31 (each warpgroup over the S^T columns it read)
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t DP_COL = 128;  // dP^T fp32; then dQ_ij [query][D] in [128, 128 + D)
  static constexpr uint32_t DK_COL = 256;  // dK [key][D]
  static constexpr uint32_t DV_COL = 256 + D;  // dV [key][D]
  static_assert(DV_COL + D <= 512, "TMEM budget");
};

// First query tile that sees key tile j (top-left causal: key k visible to query i iff k <= i).
__device__ __forceinline__ int bwd_first_q_tile(const BwdParams& p, int j) {
  return p.causal ? j : 0;
}

// Byte offset of element (row r, column c) of a 128-row tile of 16-bit values
// stored as 64-column slabs with the 128-byte swizzle (16-byte chunk index
// XOR row % 8), the layout TMA writes and the tcgen05 descriptors read.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return static_cast<uint32_t>((c >> 6) * (128 * 128) + r * 128 +
                               ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}

// ---------------------------------------------------------------------------
// prep: D = rowsum(dO * O), lse2 = lse * log2 e (padded), dq_acc = 0.
// One warp per 4 rows: 8 lanes per row, each 16 bytes (8 elements) of O and
// dO per step.
// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ o,
                                                       const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, float* lse2,
                                                       float* dsum, float* dq_acc, int Nq, int nq_pad,
                                                       long long BH) {
  const long long rows = BH * nq_pad;
  const int lane = threadIdx.x & 31;
  const int sub = lane >> 3, part = lane & 7;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long w = warp0; 4 * w < rows; w += nwarps) {
    const long long prow = 4 * w + sub;  // padded row index: bh * nq_pad + i
    float acc = 0.f;
    bool valid = false;
    long long row = 0;
    if (prow < rows) {
      const long long bh = prow / nq_pad;
      const int i = static_cast<int>(prow - bh * nq_pad);
      valid = i < Nq;
      row = bh * Nq + i;
      if (valid) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) {
          const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + c0 + part * 8);
          const uint4 b = *reinterpret_cast<const uint4*>(dout + row * D + c0 + part * 8);
          const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float a0, a1, b0, b1;
            if constexpr (BF16) {
              a0 = __uint_as_float(av[e] << 16);
              a1 = __uint_as_float(av[e] & 0xFFFF0000u);
              b0 = __uint_as_float(bv[e] << 16);
              b1 = __uint_as_float(bv[e] & 0xFFFF0000u);
            } else {
              a0 = __half2float(__ushort_as_half(static_cast<unsigned short>(av[e] & 0xFFFFu)));
              a1 = __half2float(__ushort_as_half(static_cast<unsigned short>(av[e] >> 16)));
              b0 = __half2float(__ushort_as_half(static_cast<unsigned short>(bv[e] & 0xFFFFu)));
              b1 = __half2float(__ushort_as_half(static_cast<unsigned short>(bv[e] >> 16)));
            }
            acc = fmaf(a0, b0, acc);
            acc = fmaf(a1, b1, acc);
          }
        }
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (prow < rows) {
      if (part == 0) {
        dsum[prow] = valid ? acc : 0.f;
        lse2[prow] = valid ? lse[row] * 1.4426950408889634f : INFINITY;
      }
      if (valid) {
        float4* z = reinterpret_cast<float4*>(dq_acc + row * D);
#pragma unroll
        for (int c = part; c < D / 4; c += 8) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// dq = scale * dq_acc, rounded to the input dtype.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                     uint16_t* __restrict__ dq, long long n4,
                                                     float scale) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[i];
    uint2 r;
    r.x = pack2<BF16>(a.x * scale, a.y * scale);
    r.y = pack2<BF16>(a.z * scale, a.w * scale);
    reinterpret_cast<uint2*>(dq)[i] = r;
  }
}

// ---------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using L = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + L::BAR_OFF + 8u * i; };

  // key tile j of (batch, head) bh.  Without the mask all heads' tile 0 come
  // first, so CTAs that run together add their dQ tiles into different heads;
  // under the causal mask a head's key tiles are adjacent, so the CTAs that
  // read its Q and dO run together and share them through L2 (measured: -2 %
  // and -8 % on the causal workloads, +3 % on the non-causal ones)
  int j, bh;
  if (p.causal) {
    bh = static_cast<int>(blockIdx.x / p.nk_tiles);
    j = static_cast<int>(blockIdx.x - static_cast<long long>(bh) * p.nk_tiles);
  } else {
    j = static_cast<int>(blockIdx.x / p.BH);
    bh = static_cast<int>(blockIdx.x - static_cast<long long>(j) * p.BH);
  }
  const int i0 = bwd_first_q_tile(p, j);
  const int n_tiles = p.nq_tiles > i0 ? p.nq_tiles - i0 : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::KV_FULL), 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar(L::RING_FULL + s), 1);
      mbar_init(bar(L::RING_EMPTY + s), 1);
    }
    mbar_init(bar(L::S_READY), 1);
    mbar_init(bar(L::DP_READY), 1);
    mbar_init(bar(L::P_READY), 256);
    mbar_init(bar(L::DS_READY), 256);
    mbar_init(bar(L::DQ_READY), 1);
    mbar_init(bar(L::DQ_FREE), 128);
    mbar_init(bar(L::DONE), 1);
    mbar_init(bar(L::RO_SYNC), 128);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == BWD_LOAD_WARP && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  if (warp == BWD_MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == BWD_LOAD_WARP) {
    // ------------------------------------------------------------- TMA loads
    const bool leader = elect_one();
    bool ok = true;
    if (leader) {
      mbar_arrive_expect_tx(bar(L::KV_FULL), 2 * L::TILE_BYTES);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        tma_load_3d(sbase + L::K_OFF + h * L::HALF_BYTES, &tm_k, bar(L::KV_FULL), h * 64, j * 128, bh);
        tma_load_3d(sbase + L::V_OFF + h * L::HALF_BYTES, &tm_v, bar(L::KV_FULL), h * 64, j * 128, bh);
      }
    }
    __syncwarp();
    int n = 0;
    for (; ok && n < n_tiles; ++n) {
      const int s = n % L::STAGES;
      if (n >= L::STAGES) {
        ok = __all_sync(0xffffffffu, wait_phase(bar(L::RING_EMPTY + s), (n / L::STAGES - 1) & 1,
                                                abort_flag, SITE_LOAD_KV_EMPTY));
        if (!ok) break;
      }
      if (leader) {
        const int q0 = (i0 + n) * 128;
        const uint32_t dst = sbase + L::RING_OFF + s * 2 * L::TILE_BYTES;
        mbar_arrive_expect_tx(bar(L::RING_FULL + s),
                              2 * L::TILE_BYTES + (L::STATS_IN_SMEM ? 1024 : 0));
        if constexpr (L::STATS_IN_SMEM) {
          const size_t row0 = static_cast<size_t>(bh) * p.nq_pad + q0;  // 512-byte aligned
          bulk_load(sbase + L::STATS_OFF + s * 1024, p.lse2 + row0, 512, bar(L::RING_FULL + s));
          bulk_load(sbase + L::STATS_OFF + s * 1024 + 512, p.dsum + row0, 512,
                    bar(L::RING_FULL + s));
        }
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(dst + h * L::HALF_BYTES, &tm_q, bar(L::RING_FULL + s), h * 64, q0, bh);
          tma_load_3d(dst + L::TILE_BYTES + h * L::HALF_BYTES, &tm_do, bar(L::RING_FULL + s), h * 64,
                      q0, bh);
        }
      }
      __syncwarp();
    }
    // every issued load must land before the CTA exits
    wait_phase(bar(L::KV_FULL), 0, abort_flag, SITE_DRAIN, false);
    for (int m = n > L::STAGES ? n - L::STAGES : 0; m < n; ++m)
      wait_phase(bar(L::RING_FULL + m % L::STAGES), (m / L::STAGES) & 1, abort_flag, SITE_DRAIN,
                 false);
    __syncwarp();
  } else if (warp == BWD_MMA_WARP) {
    // ------------------------------------------------------------- MMA issue
    const bool leader = elect_one();
    constexpr uint32_t IDESC_SS = idesc_f16(BF16, false, false, 128, 128);  // S^T, dP^T
    constexpr uint32_t IDESC_KB = idesc_f16(BF16, false, true, 128, D);     // dV, dK: B MN-major
    constexpr uint32_t IDESC_QA = idesc_f16(BF16, true, true, 128, D);      // dQ: A, B MN-major
    // K-major descriptors (head dim contiguous; k-step = 16 elements = 32 bytes
    // within a 128-byte row, the next 64 columns one slab on)
    const uint64_t k_kmaj = sw128_desc(sbase + L::K_OFF, 16, 1024);
    const uint64_t v_kmaj = sw128_desc(sbase + L::V_OFF, 16, 1024);
    const uint64_t ring_kmaj = sw128_desc(sbase + L::RING_OFF, 16, 1024);
    const uint64_t ds_kmaj = sw128_desc(sbase + L::DS_OFF, 16, 1024);
    // MN-major descriptors (rows are the K dimension: 8-row groups 1 KB apart,
    // a k-step of 16 rows = 2 KB; 64-column slabs 16 KB apart)
    const uint64_t ring_mn = sw128_desc(sbase + L::RING_OFF, L::HALF_BYTES, 1024);
    const uint64_t k_mn = sw128_desc(sbase + L::K_OFF, L::HALF_BYTES, 1024);
    const uint64_t ds_mn = sw128_desc(sbase + L::DS_OFF, L::HALF_BYTES, 1024);
    const uint32_t t_s = tmem_base + L::S_COL, t_dp = tmem_base + L::DP_COL;
    const uint32_t t_dk = tmem_base + L::DK_COL, t_dv = tmem_base + L::DV_COL;
    constexpr uint32_t TILE16 = L::TILE_BYTES >> 4;
    auto kstep_kmaj = [](int kk) -> uint32_t {
      return static_cast<uint32_t>(((kk / 4) * L::HALF_BYTES + (kk % 4) * 32) >> 4);
    };
    // X^T = A * B^T with A the resident K or V tile, B the stage's Q or dO tile
    auto issue_st = [&](uint32_t dst, uint64_t a, uint64_t b) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(dst, a + kstep_kmaj(kk), b + kstep_kmaj(kk), IDESC_SS, kk > 0 ? 1u : 0u);
    };
    bool ok = __all_sync(0xffffffffu, wait_phase(bar(L::KV_FULL), 0, abort_flag, SITE_MMA_KV_FULL));
    if (ok && n_tiles > 0) {
      ok = __all_sync(0xffffffffu, wait_phase(bar(L::RING_FULL), 0, abort_flag, SITE_MMA_Q_FULL));
      if (ok) {
        tc_fence_after();
        if (leader) {
          issue_st(t_s, k_kmaj, ring_kmaj);  // S^T(0) = K_j Q_i0^T
          mma_commit(bar(L::S_READY));
        }
        __syncwarp();
      }
    }
    for (int n = 0; ok && n < n_tiles; ++n) {
      const int s = n % L::STAGES;
      const uint32_t q16 = s * 2 * TILE16, do16 = q16 + TILE16;
      // dP^T(n) = V_j dO_i^T, into the columns the readout of dQ(n - 1) frees
      if (n > 0) {
        ok = __all_sync(0xffffffffu, wait_phase(bar(L::DQ_FREE), (n - 1) & 1, abort_flag,
                                                SITE_MMA_P_FULL));
        if (!ok) break;
      }
      tc_fence_after();
      if (leader) {
        issue_st(t_dp, v_kmaj, ring_kmaj + do16);
        mma_commit(bar(L::DP_READY));
      }
      __syncwarp();
      // dV += P^T dO_i (P^T from TMEM, 16 queries = 8 columns per k-step;
      // queries 64 w .. 64 w + 63 at columns 64 w .. 64 w + 31)
      ok = __all_sync(0xffffffffu, wait_phase(bar(L::P_READY), n & 1, abort_flag, SITE_MMA_P_FULL));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(t_dv, t_s + (kk >> 2) * 64 + (kk & 3) * 8, ring_mn + do16 + kk * (2048 >> 4),
                 IDESC_KB, (n > 0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
      // S^T(n + 1): queued behind dV(n), which reads the P^T it overwrites
      if (n + 1 < n_tiles) {
        const int s1 = (n + 1) % L::STAGES;
        ok = __all_sync(0xffffffffu, wait_phase(bar(L::RING_FULL + s1), ((n + 1) / L::STAGES) & 1,
                                                abort_flag, SITE_MMA_Q_FULL));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          issue_st(t_s, k_kmaj, ring_kmaj + s1 * 2 * TILE16);
          mma_commit(bar(L::S_READY));
        }
        __syncwarp();
      }
      // dK += dS^T Q_i and dQ_ij = dS K_j (dS^T from shared memory)
      ok = __all_sync(0xffffffffu, wait_phase(bar(L::DS_READY), n & 1, abort_flag, SITE_MMA_P_FULL));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(t_dk, ds_kmaj + kstep_kmaj(kk), ring_mn + q16 + kk * (2048 >> 4), IDESC_KB,
                 (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(t_dp, ds_mn + kk * (2048 >> 4), k_mn + kk * (2048 >> 4), IDESC_QA,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar(L::DQ_READY));
        if (!L::DQ_IN_STAGE) mma_commit(bar(L::RING_EMPTY + s));  // else the readout frees it
      }
      __syncwarp();
    }
    if (leader) mma_commit(bar(L::DONE));
    __syncwarp();
    wait_phase(bar(L::DONE), 0, abort_flag, SITE_DRAIN, false);
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------------------------------------- dQ readout
    const int r = (warp - 8) * 32 + lane;  // query row within the tile
    const uint32_t t_dq = tmem_base + L::DP_COL + (static_cast<uint32_t>((warp - 8) * 32) << 16);
    const bool issuer = (threadIdx.x == 8 * 32);  // issues and waits for the bulk reductions
    uint32_t ro_phase = 0;
    auto ro_sync = [&]() -> bool {  // bounded rendezvous of the 128 readout threads
      mbar_arrive(bar(L::RO_SYNC));
      const bool ok = wait_phase(bar(L::RO_SYNC), ro_phase, abort_flag, SITE_SOFTMAX_SYNC);
      ro_phase ^= 1;
      return __all_sync(0xffffffffu, ok);
    };
    for (int n = 0; n < n_tiles; ++n) {
      const bool ok = __all_sync(0xffffffffu, wait_phase(bar(L::DQ_READY), n & 1, abort_flag,
                                                         SITE_SOFTMAX_O_READY));
      if (!ok) break;
      tc_fence_after();
      const int q0 = (i0 + n) * 128;
      if constexpr (!L::DQ_IN_STAGE) {
        uint32_t v[64];
        tmem_ld32(t_dq, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(t_dq + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_wait_ld_regs(v);
        tc_fence_before();
        mbar_arrive(bar(L::DQ_FREE));
        // slot n & 1 was last read by the reductions of tile n - 2
        if (issuer && n >= 2) bulk_wait_group_read<1>();
        if (!ro_sync()) break;
        uint8_t* slot = smem + L::DQ_OFF + (n & 1) * 32768;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(slot + h * 16384 + r * 128 + ((ch ^ (r & 7)) << 4)) =
                make_uint4(v[32 * h + 4 * ch], v[32 * h + 4 * ch + 1], v[32 * h + 4 * ch + 2],
                           v[32 * h + 4 * ch + 3]);
        fence_proxy_async_shared();
        if (!ro_sync()) break;
        if (issuer) {
          // rows past Nq fall outside the tensor and are not written
          tma_reduce_add_3d(&tm_dq, sbase + L::DQ_OFF + (n & 1) * 32768, 0, q0, bh);
          tma_reduce_add_3d(&tm_dq, sbase + L::DQ_OFF + (n & 1) * 32768 + 16384, 32, q0, bh);
          bulk_commit_group();
        }
      } else {
        // stage the tile in the ring stage of tile n (free: DQ_READY(n) follows
        // every MMA of tile n), four 32-column boxes of 16 KB
        const int s = n % L::STAGES;
        uint8_t* stage = smem + L::RING_OFF + s * 2 * L::TILE_BYTES;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) {
          uint32_t v[64];
          tmem_ld32(t_dq + c0, *reinterpret_cast<uint32_t(*)[32]>(v));
          tmem_ld32(t_dq + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          tmem_wait_ld_regs(v);
          if (c0 + 64 == D) {
            tc_fence_before();
            mbar_arrive(bar(L::DQ_FREE));
          }
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              *reinterpret_cast<uint4*>(stage + (c0 / 32 + h) * 16384 + r * 128 +
                                        ((ch ^ (r & 7)) << 4)) =
                  make_uint4(v[32 * h + 4 * ch], v[32 * h + 4 * ch + 1], v[32 * h + 4 * ch + 2],
                             v[32 * h + 4 * ch + 3]);
        }
        fence_proxy_async_shared();
        if (!ro_sync()) break;
        if (issuer) {
          const uint32_t src = sbase + L::RING_OFF + s * 2 * L::TILE_BYTES;
#pragma unroll
          for (int b = 0; b < D / 32; ++b) tma_reduce_add_3d(&tm_dq, src + b * 16384, 32 * b, q0, bh);
          bulk_commit_group();
          bulk_wait_group_read<0>();  // the stage has been read: the loader may refill it
          mbar_arrive(bar(L::RING_EMPTY + s));
        }
      }
    }
    if (issuer) bulk_wait_group<0>();  // every reduction done before the CTA exits
  } else {
    // ------------------------------------------------------------- softmax
    // Thread = key row r of the tile; warpgroup w takes query columns
    // [64 w, 64 w + 64).  Every step is elementwise: lse and D are known.
    const int w = warp / 4;
    const int r = (warp % 4) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t t_s = tmem_base + lane_off + L::S_COL;
    const uint32_t t_dp = tmem_base + lane_off + L::DP_COL;
    const int key = j * 128 + r;
    const bool key_ok = key < p.Nk;
    const float sl2 = p.scale_log2;
    uint8_t* ds_tile = smem + L::DS_OFF;
    const float* lse2_bh = p.lse2 + static_cast<size_t>(bh) * p.nq_pad;
    const float* dsum_bh = p.dsum + static_cast<size_t>(bh) * p.nq_pad;
    const float* stats_smem = reinterpret_cast<const float*>(smem + L::STATS_OFF);
    bool ok = true;
    for (int n = 0; ok && n < n_tiles; ++n) {
      const int q0 = (i0 + n) * 128;
      const int qw = q0 + 64 * w;  // first query of this warpgroup's columns
      // d = 128: lane l holds the lse2 and D of queries qw + l and qw + 32 + l
      // (coalesced loads issued before the wait); column c is then taken from
      // lane c % 32 by a shuffle
      float lse_lo = 0.f, lse_hi = 0.f, ds_lo = 0.f, ds_hi = 0.f;
      if constexpr (!L::STATS_IN_SMEM) {
        lse_lo = lse2_bh[qw + lane];
        lse_hi = lse2_bh[qw + 32 + lane];
        ds_lo = dsum_bh[qw + lane];
        ds_hi = dsum_bh[qw + 32 + lane];
      }
      // d = 64: the stage's lse2 / D landed with Q_i; these threads observe
      // that stage's completed phase themselves before reading them (the
      // stage is refilled only after this tile's dS is handed over, so the
      // phase is unambiguous; S^T(n) is computed from the same stage).  The
      // first lse2 values are loaded before the S wait and each later one
      // four float4 ahead of its use, so no exponential waits on a load.
      const float* stage_stats = stats_smem + (n % L::STAGES) * 256;
      const float4* l4 = reinterpret_cast<const float4*>(stage_stats + 64 * w);
      float4 lq[4];
      if constexpr (L::STATS_IN_SMEM) {
        ok = __all_sync(0xffffffffu, wait_phase(bar(L::RING_FULL + n % L::STAGES),
                                                (n / L::STAGES) & 1, abort_flag,
                                                SITE_SOFTMAX_S_FULL));
        if (!ok) break;
#pragma unroll
        for (int i = 0; i < 4; ++i) lq[i] = l4[i];
      }
      ok = __all_sync(0xffffffffu, wait_phase(bar(L::S_READY), n & 1, abort_flag,
                                              SITE_SOFTMAX_S_FULL));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(t_s + 64 * w, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(t_s + 64 * w + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_wait_ld_regs(sr);
      // P = 2^(s * scale * log2 e - lse2); 0 for keys past Nk, queries past
      // Nq (lse2 = +inf there) and, causal, queries before the key
      uint32_t pk[32];
      const bool diag = p.causal && qw < key;  // some of these queries precede the key
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        float lsv[4];
        if constexpr (L::STATS_IN_SMEM) {
          const float4 lv = lq[c4 % 4];
          if (c4 + 4 < 16) lq[c4 % 4] = l4[c4 + 4];
          lsv[0] = lv.x;
          lsv[1] = lv.y;
          lsv[2] = lv.z;
          lsv[3] = lv.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            lsv[e] = __shfl_sync(0xffffffffu, c4 < 8 ? lse_lo : lse_hi, (4 * c4 + e) & 31);
        }
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * c4 + e;
          float x = fmaf(__uint_as_float(sr[c]), sl2, -lsv[e]);
          if (!key_ok || (diag && qw + c < key)) x = -INFINITY;
          pv[e] = ex2_approx(x);
        }
        pk[2 * c4] = pack2<BF16>(pv[0], pv[1]);
        pk[2 * c4 + 1] = pack2<BF16>(pv[2], pv[3]);
      }
      // over this warpgroup's own S^T columns, which only it has read
      tmem_st16(t_s + 64 * w, *reinterpret_cast<uint32_t(*)[16]>(pk));
      tmem_st16(t_s + 64 * w + 16, *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::P_READY));
      // dS = P (dP - D), from the rounded P the dV product used; the D values
      // are loaded ahead of their use like lse2
      const float4* d4 = reinterpret_cast<const float4*>(stage_stats + 128 + 64 * w);
      float4 dq4[4];
      if constexpr (L::STATS_IN_SMEM) {
#pragma unroll
        for (int i = 0; i < 4; ++i) dq4[i] = d4[i];
      }
      ok = __all_sync(0xffffffffu, wait_phase(bar(L::DP_READY), n & 1, abort_flag,
                                              SITE_SOFTMAX_S_FULL));
      if (!ok) break;
      if (n > 0) {  // dK and dQ of the previous tile have read the dS^T tile
        ok = __all_sync(0xffffffffu, wait_phase(bar(L::DQ_READY), (n - 1) & 1, abort_flag,
                                                SITE_SOFTMAX_O_READY));
        if (!ok) break;
      }
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t dp[32];
        tmem_ld32(t_dp + 64 * w + 32 * half, dp);
        tmem_wait_ld_regs(dp);
        uint32_t ds[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          float dsv[4];
          if constexpr (L::STATS_IN_SMEM) {
            const int di = 8 * half + c4;
            const float4 dv = dq4[di % 4];
            if (di + 4 < 16) dq4[di % 4] = d4[di + 4];
            dsv[0] = dv.x;
            dsv[1] = dv.y;
            dsv[2] = dv.z;
            dsv[3] = dv.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dsv[e] = __shfl_sync(0xffffffffu, half ? ds_hi : ds_lo, (4 * c4 + e) & 31);
          }
          float o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 32 * half + 4 * c4 + e;  // column within this warpgroup's 64
            const uint32_t pw = pk[c >> 1];
            const float pf = BF16 ? __uint_as_float((c & 1) ? (pw & 0xFFFF0000u) : (pw << 16))
                                  : __half2float(__ushort_as_half(
                                        static_cast<unsigned short>((c & 1) ? (pw >> 16) : (pw & 0xFFFFu))));
            o[e] = pf * (__uint_as_float(dp[4 * c4 + e]) - dsv[e]);
          }
          ds[2 * c4] = pack2<BF16>(o[0], o[1]);
          ds[2 * c4 + 1] = pack2<BF16>(o[2], o[3]);
        }
        // 32 queries = four 16-byte chunks of row r of the swizzled dS^T tile
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int col = 64 * w + 32 * half + 8 * ch;
          *reinterpret_cast<uint4*>(ds_tile + sw128_offset(r, col)) =
              make_uint4(ds[4 * ch], ds[4 * ch + 1], ds[4 * ch + 2], ds[4 * ch + 3]);
        }
      }
      fence_proxy_async_shared();
      tc_fence_before();
      mbar_arrive(bar(L::DS_READY));
    }
    // ----------------------------------------------------------- epilogue
    // warpgroup 0 writes dK (times scale), warpgroup 1 dV; rows < Nk
    if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar(L::DONE), 0, abort_flag, SITE_DRAIN));
    if (ok) {
      tc_fence_after();
      const uint32_t t_acc = tmem_base + lane_off + (w == 0 ? L::DK_COL : L::DV_COL);
      const float mul = w == 0 ? p.scale : 1.f;
      uint16_t* out = reinterpret_cast<uint16_t*>(w == 0 ? p.dk : p.dv);
      uint4* orow = reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * p.Nk + key) * D);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t a[32];
        tmem_ld32(t_acc + c0, a);
        tmem_wait_ld_regs(a);
        uint32_t pk2[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk2[i] = n_tiles > 0 ? pack2<BF16>(__uint_as_float(a[2 * i]) * mul,
                                             __uint_as_float(a[2 * i + 1]) * mul)
                               : 0u;  // no query sees this key tile: zero gradient
        if (key_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            orow[c0 / 8 + v4] = make_uint4(pk2[4 * v4], pk2[4 * v4 + 1], pk2[4 * v4 + 2], pk2[4 * v4 + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BWD_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace attn_sm100
