// Exact attention forward for sm_100a (B200):
//   O = softmax(Q K^T * scale [+ top-left causal mask]) V,   lse = m + ln(l)
//
// The method is the tiled online softmax of the pages: "FlashAttention 深度解读"
// (coreui.cn), section "原理" (block tiling plus online softmax kept as a
// running max and exponent sum) and section "实现 3" (subtract the running
// max before exponentiating); YOLO11 x FlashAttention-2 (kwkr.cn), section
// 1.2 (rescale the accumulated output whenever a new block raises the max;
// split work over sequence blocks, heads and batch).  The N x N score
// matrix never leaves the SM: S lives in tensor memory (TMEM) one 128 x 128
// tile at a time.
//
// Blackwell mapping (one CTA per SM, persistent over work units):
//   * a work unit is two 128-row Q tiles of one (batch, head) that share
//     every K/V tile the CTA loads (a dual unit: the last tiles of two heads,
//     each with its own K/V stream); causal units pair a heavy query pair
//     with its light mirror; split mode shares a ragged grid's key-tile steps
//     out evenly and merges the pieces in the log domain;
//   * warp 9 issues the TMA loads of the unit's Q tiles and of K_j into a
//     ring of K slots, warp 11 those of V_j into a ring of V slots, each slot
//     guarded by a full / empty mbarrier pair (128-byte swizzle; every CTA
//     loads its own tiles);
//   * warp 8 issues tcgen05.mma S = Q_t K_j^T (fp32) into one of NSB TMEM S/P
//     buffers as soon as K_j is in and the buffer's last P V is done, so it
//     runs ahead of the softmax; warp 10 issues O_t += P V_j with P read from
//     TMEM, where the softmax wrote it over S as 16-bit pairs (at d = 128,
//     with two buffers, warp 8 issues both in sequence order).  The producer
//     warps loop on all lanes and one elected lane issues; tcgen05.commit
//     signals the softmax warps and releases ring slots;
//   * warps 0-3 own Q tile 0 and warps 4-7 Q tile 1, one thread per query
//     row: each reads its S row from TMEM, masks, keeps the running max m
//     (base 2, pre-multiplied by scale * log2 e) and sum l, writes P, and
//     rescales its O row in TMEM by 2^(m_old - m_new) when the max rose by
//     more than the lazy threshold.  While one warpgroup runs its softmax the
//     tensor core works on the other tile, so exponentials and MMAs overlap;
//   * the epilogue divides O by l, rounds to the input dtype and stores the
//     rows below Nq; lse = (m + log2 l) * ln 2.
//
// Every mbarrier wait is bounded (about one second of %globaltimer); on
// timeout the kernel records where in a device status word, tells the other
// roles to stop, waits (bounded) for its own TMA loads and MMAs to land,
// frees TMEM and returns.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int BLOCK_M = 128;     // query rows per Q tile (= TMEM lanes)
constexpr int BLOCK_N = 128;     // keys per K / V tile
// 12 warps = 3 warpgroups: two softmax warpgroups (warps 0-3, 4-7) and one
// producer warpgroup (warp 8 issues the S MMAs, warp 9 the TMA loads of Q and
// K, warp 10 the P V MMAs, warp 11 the TMA loads of V).  Launched at 168
// registers per thread (the per-SM-sub-partition limit for 3 warps each); the
// producer warpgroup then gives registers up and the softmax warpgroups take
// them (2 * 128 * 200 + 128 * 96 = 63488, or 2 * 128 * 208 + 128 * 88 =
// 64512, both <= 384 * 168), so the increase never waits on registers that
// do not exist.  At 96 the MMA issuers of the unit-mode kernels keep one
// descriptor word in local memory (an L1 hit per MMA issue, off the softmax's
// critical path); giving them 104 removes that spill but measured 2-7 %
// slower.
constexpr int NUM_THREADS = 384;
constexpr int MMA_WARP = 8;    // issues S = Q K^T
constexpr int LOAD_WARP = 9;   // TMA loads of Q and K
constexpr int PV_WARP = 10;    // issues O += P V
constexpr int VLOAD_WARP = 11; // TMA loads of V
// The split-mode kernel (piece bookkeeping and merge in the softmax) needs a
// few more softmax registers than the unit-mode one.
template <bool SPLIT>
__host__ __device__ constexpr uint32_t softmax_regs() { return SPLIT ? 208 : 200; }
template <bool SPLIT>
__host__ __device__ constexpr uint32_t producer_regs() { return SPLIT ? 88 : 96; }
static_assert(2 * 128 * softmax_regs<true>() + 128 * producer_regs<true>() <= NUM_THREADS * 168,
              "register split exceeds the launch budget");
static_assert(2 * 128 * softmax_regs<false>() + 128 * producer_regs<false>() <= NUM_THREADS * 168,
              "register split exceeds the launch budget");
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr float RESCALE_LOG2 = 8.0f;  // lazy-rescale threshold for the running max
// Of every 16 key pairs in a 32-key chunk, this many take 2^x from a
// polynomial on the FMA pipe and the rest from the MUFU ex2 unit, so the two
// pipes share the exponentials.  At d = 64 the MUFU bounds the softmax; at
// d = 128 the tensor core does, and the polynomial only costs issue slots --
// except with e4m3 operands, whose MMAs take half the time, so the MUFU
// bounds that softmax as well.
template <int D, bool FP8 = false>
__host__ __device__ constexpr int exp_poly_pairs() { return (D == 64 || FP8) ? 4 : 0; }

// Device status word: 0 = healthy; otherwise 0x80000000 | site.
__device__ unsigned int g_attn_status = 0;

enum WaitSite : uint32_t {
  SITE_LOAD_Q_EMPTY = 1,
  SITE_LOAD_KV_EMPTY = 2,
  SITE_MMA_Q_FULL = 3,
  SITE_MMA_KV_FULL = 4,
  SITE_MMA_P_FULL = 5,
  SITE_SOFTMAX_S_FULL = 6,
  SITE_SOFTMAX_O_READY = 7,
  SITE_DRAIN = 8,
  SITE_SOFTMAX_SYNC = 9,
  SITE_INJECTED = 10,  // a wait made unsatisfiable on purpose (attn_fwd_stall_test)
};

// Test hook: which role waits on a barrier nothing ever arrives on.
enum StallSite : int {
  STALL_NONE = 0,
  STALL_SOFTMAX = 1,     // softmax warpgroup 0, before its first score tile
  STALL_MMA = 2,         // the S-issuing MMA warp, before its first MMA
  STALL_LOAD = 3,        // the K/Q TMA warp, before its first load
  STALL_SPLIT_SYNC = 4,  // softmax warpgroup 0, before the split-piece rendezvous
};

struct FwdParams {
  void* o;         // [B, H, Nq, D] fp16 / bf16
  float* lse;      // [B, H, Nq] fp32, or nullptr
  int Nq, Nk, BH;
  int num_q_pairs;  // ceil(ceil(Nq / 128) / 2)
  int num_kv_tiles; // ceil(Nk / 128)
  int units_per_head; // causal: ceil(num_q_pairs / 2); dual units: num_q_tiles / 2; else num_q_pairs
  int num_units;    // BH * units_per_head (+ the dual units)
  // Dual units (non-causal unit mode, odd query-tile count): units from
  // dual_base on pair the lone last query tile (rows last_q0..) of two heads;
  // -1 when there are none.
  int dual_base;
  int last_q0;
  int causal;
  float scale_log2; // scale * log2(e) (e4m3 operands: times the Q and K descales)
  float o_scale;    // e4m3 operands: the V descale, applied with 1 / l; unused otherwise
  // Split mode.  Every unit is one query pair of one (batch, head); its key
  // tiles are flattened into total_steps = B H * steps_per_head steps (a
  // pair needs num_kv_tiles of them, or under the causal mask only the tiles
  // its later query tile sees) and CTA c takes steps
  // [c * total_steps / grid, (c + 1) * total_steps / grid), so every CTA does
  // the same work however the units divide.  A unit cut by a range boundary
  // is computed in pieces; each piece leaves its normalised O and lse in the
  // caller's workspace and the last piece to finish merges them.
  int split;
  int num_q_tiles;         // ceil(Nq / 128)
  long long steps_per_head;
  long long total_steps;
  float* ws_o;           // [grid][2 slots][2 tiles][128 rows][D]
  float* ws_lse;         // [grid][2 slots][2 tiles][128 rows]
  unsigned int* ws_count;  // [num_units] pieces finished; zero between calls
  int stall_site;          // StallSite; 0 except through the test hook
};

// FP8: e4m3 operands (d = 128 only).  A tile row is then 128 one-byte
// elements, one 128-byte swizzle row, and V arrives transposed (Vt tiles of
// d rows x 128 keys), so both MMAs read K-major operands.
template <int D, bool FP8 = false>
struct SmemLayout {
  // one 128-row slab of 128-byte rows, 128-byte swizzled: 64 fp16 / bf16 or 128 e4m3 columns
  static constexpr int HALF_BYTES = BLOCK_M * 128;
  static constexpr int HALVES = FP8 ? 1 : D / 64;
  static_assert(!FP8 || D == 128, "e4m3 tiles hold 128 one-byte columns");
  static constexpr int TILE_BYTES = HALVES * HALF_BYTES;
  // separate K and V rings, filled in the order the MMA warp consumes them
  static constexpr int K_STAGES = (D == 64 || FP8) ? 4 : 3;
  static constexpr int V_STAGES = (D == 64 || FP8) ? 4 : 2;
  // Q: slots of two tiles.  Two slots at d = 64 and with e4m3 tiles, so the
  // next item's Q tiles load while the current item runs and its first S
  // does not wait for them; one at d = 128 (16-bit), where shared memory has
  // no room for a second.
  static constexpr int Q_SLOTS = (D == 64 || FP8) ? 2 : 1;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_SLOTS * 2 * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + K_STAGES * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + V_STAGES * TILE_BYTES;
  // S/P buffers in TMEM: three at d = 64 (so a tile's next S is computed
  // while its current P is still being written), two at d = 128 (TMEM holds
  // 2 x 128 S columns + 2 x 128 O columns and nothing more).
  static constexpr int NSB = (D == 64) ? 3 : 2;
  // mbarrier indices
  static constexpr int K_FULL = 0;
  static constexpr int K_EMPTY = K_FULL + K_STAGES;
  static constexpr int V_FULL = K_EMPTY + K_STAGES;
  static constexpr int V_EMPTY = V_FULL + V_STAGES;
  static constexpr int Q_FULL = V_EMPTY + V_STAGES;  // + slot
  static constexpr int Q_EMPTY = Q_FULL + Q_SLOTS;   // + slot
  // S ready: one barrier per (buffer, tile), so each softmax warpgroup only
  // waits on phases it alone consumes (a per-buffer barrier shared by both
  // tiles could be two phases behind a warpgroup that skipped an item).
  static constexpr int S_FULL = Q_EMPTY + Q_SLOTS;  // + 2 * buffer + tile
  static constexpr int P_FULL = S_FULL + 2 * NSB;  // + buffer (one waiter: the MMA warp)
  static constexpr int O_READY = P_FULL + NSB; // + tile: one phase per P V MMA of the tile
  static constexpr int PV_DONE = O_READY + 2;  // + buffer: P V of that buffer finished
  static constexpr int DRAIN = PV_DONE + NSB;  // + 0 (S warp), + 1 (P V warp)
  static constexpr int SYNC = DRAIN + 2;        // rendezvous of the 256 softmax threads
  static constexpr int NEVER = SYNC + 1;        // no thread ever arrives (test hook)
  static constexpr int NUM_BARS = NEVER + 1;
  // TMEM address, abort flag, split flag, then (d = 64) the P V MMAs completed
  // per tile, published by the P V issuer
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int PV_DONE_OFF = MISC_OFF + 16;
  static constexpr int BYTES = PV_DONE_OFF + 8 + 1024;  // + slack to align the base to 1 KB
  // TMEM columns (512 allocated): S/P buffers, then O of tile 0 and tile 1
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;           // + 128 * buffer
  static constexpr uint32_t O_COL = 128 * NSB;   // + D * tile
  static_assert(O_COL + 2 * D <= TMEM_COLS, "TMEM budget");
};

struct Unit {
  int bh;     // (batch, head) of tile 0
  int q0;     // first query row of tile 0
  int bh1;    // (batch, head) of tile 1: bh, except in a dual unit
  int q1;     // first query row of tile 1: q0 + 128, except in a dual unit
  int kvs;    // K (and V) tiles per key step: 1 (shared by both tiles) or 2 (dual unit)
  int jbase;  // first K/V tile of this item (non-zero only for split pieces)
  int n[2];   // K/V tiles each Q tile visits from jbase (0 = tile lies past Nq)
  int nmax;
  int unit, piece, pieces, c_first;  // split pieces: which, how many, CTA of piece 0
};

// Work schedule.  A work unit belongs to one (batch, head) and holds one or
// two "items"; an item is a pair of adjacent 128-row Q tiles.  CTA c takes
// units c, c + grid, c + 2 grid, ...; consecutive units belong to the same
// head, so CTAs running at the same time share that head's K/V through L2.
//   non-causal: one item per unit, every item costs the same.  With an odd
//     number of query tiles each head's last tile has no partner; those
//     tiles are paired across heads (tile 0 from head 2d, tile 1 from head
//     2d + 1) in "dual" units placed after all the others, so no warpgroup
//     idles through a unit.  A dual unit streams both heads' K and V.
//   causal: unit b of a head holds Q pair (n_pairs - 1 - b) and its mirror b,
//     heaviest first; the two together always visit about n_pairs + 1 K/V
//     tiles, so every unit costs the same and the persistent CTAs finish
//     together.
__device__ __forceinline__ int unit_items(const FwdParams& p, int u) {
  if (!p.causal) return 1;
  const int b = u % p.units_per_head;
  return (b != p.num_q_pairs - 1 - b) ? 2 : 1;
}

// PLAIN: unit b of a head is query pair b (split mode), without the causal
// heavy / light pairing.
template <bool DUAL, bool PLAIN = false>
__device__ __forceinline__ Unit decode_item(const FwdParams& p, int u, int item) {
  Unit w;
  w.jbase = 0;
  w.unit = u;
  w.piece = 0;
  w.pieces = 1;
  w.c_first = 0;
  if (DUAL && u >= p.dual_base) {
    const int h0 = 2 * (u - p.dual_base);
    const bool pair = h0 + 1 < p.BH;
    w.bh = h0;
    w.bh1 = pair ? h0 + 1 : h0;
    w.q0 = w.q1 = p.last_q0;
    w.n[0] = p.num_kv_tiles;
    w.n[1] = pair ? p.num_kv_tiles : 0;
    w.nmax = p.num_kv_tiles;
    w.kvs = pair ? 2 : 1;
    return w;
  }
  int qp;
  w.bh = u / p.units_per_head;
  const int b = u % p.units_per_head;
  if (p.causal && !PLAIN) {
    qp = item == 0 ? p.num_q_pairs - 1 - b : b;
  } else {
    qp = b;
  }
  w.q0 = qp * 2 * BLOCK_M;
  w.bh1 = w.bh;
  w.q1 = w.q0 + BLOCK_M;
  w.kvs = 1;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qs = w.q0 + t * BLOCK_M;
    int n;
    if (qs >= p.Nq) {
      n = 0;
    } else if (p.causal) {
      const int last_row = min(qs + BLOCK_M - 1, p.Nq - 1);
      n = min(p.num_kv_tiles, last_row / BLOCK_N + 1);
    } else {
      n = p.num_kv_tiles;
    }
    w.n[t] = n;
  }
  w.nmax = max(w.n[0], w.n[1]);
  return w;
}

// Split-mode step counts.  Query tile i sees min(nk, i + 1) key tiles under
// the top-left causal mask (its last row is min(128 i + 127, Nq - 1)), so
// pair qp needs min(nk, 2 qp + 2) steps, or min(nk, 2 qp + 1) when its second
// tile lies past Nq; without the mask every pair needs nk.
__device__ __forceinline__ int split_unit_steps(const FwdParams& p, int qp) {
  if (!p.causal) return p.num_kv_tiles;
  const int last_tile = (2 * qp + 1 < p.num_q_tiles) ? 2 * qp + 1 : 2 * qp;
  return min(p.num_kv_tiles, last_tile + 1);
}
// Steps of the pairs before qp in a head (qp <= num_q_pairs - 1, so only
// whole pairs): sum of min(nk, 2 q + 2) over q < qp = m (m + 1) + (qp - m) nk
// with m = min(qp, nk / 2), the pairs whose count is not capped at nk.
__device__ __forceinline__ long long split_head_prefix(const FwdParams& p, int qp) {
  const long long nk = p.num_kv_tiles;
  if (!p.causal) return static_cast<long long>(qp) * nk;
  const long long m = min(static_cast<long long>(qp), nk / 2);
  return m * (m + 1) + (qp - m) * nk;
}
// The pair whose steps contain step `rem` of a head (the inverse of the prefix).
__device__ __forceinline__ int split_locate_pair(const FwdParams& p, long long rem) {
  const long long nk = p.num_kv_tiles;
  long long qp;
  if (!p.causal) {
    qp = rem / nk;
  } else {
    const long long a = nk / 2;
    if (rem < a * (a + 1)) {
      // largest m with m (m + 1) <= rem, then corrected for rounding
      long long m = static_cast<long long>((sqrt(4.0 * static_cast<double>(rem) + 1.0) - 1.0) * 0.5);
      while (m > 0 && m * (m + 1) > rem) --m;
      while ((m + 1) * (m + 2) <= rem) ++m;
      qp = m;
    } else {
      qp = a + (rem - a * (a + 1)) / nk;
    }
  }
  return static_cast<int>(min(qp, static_cast<long long>(p.num_q_pairs - 1)));
}
// First flattened step of split unit u (= bh * num_q_pairs + qp).
__device__ __forceinline__ long long split_unit_start(const FwdParams& p, int u) {
  const int bh = u / p.num_q_pairs;
  return static_cast<long long>(bh) * p.steps_per_head +
         split_head_prefix(p, u - bh * p.num_q_pairs);
}
__device__ __forceinline__ int split_locate_unit(const FwdParams& p, long long step) {
  const long long bh = step / p.steps_per_head;
  return static_cast<int>(bh) * p.num_q_pairs +
         split_locate_pair(p, step - bh * p.steps_per_head);
}

// Iterates the items of this CTA, identically in every role.
template <bool SPLIT, bool DUAL>
struct WorkCursor {
  int u, item, items;
  // split mode: this CTA's units u .. u_last, the first starting at key tile
  // j_first, the last ending before key tile j_end; pieces of the first and
  // last unit (every unit in between lies wholly inside the range)
  int u_last, j_first, j_end;
  int piece_first, pieces_first, c_first_first;
  int piece_last, pieces_last, c_first_last;
  __device__ __forceinline__ explicit WorkCursor(const FwdParams& p) {
    if constexpr (SPLIT) {
      // the 64-bit divisions run once per CTA, not once per item
      const long long begin = p.total_steps * blockIdx.x / gridDim.x;
      const long long end = p.total_steps * (blockIdx.x + 1) / gridDim.x;
      item = items = 0;
      if (begin >= end) {
        u = 0;
        u_last = -1;
        return;
      }
      u = split_locate_unit(p, begin);
      j_first = static_cast<int>(begin - split_unit_start(p, u));
      u_last = split_locate_unit(p, end - 1);
      j_end = static_cast<int>(end - split_unit_start(p, u_last));
      pieces_of(p, u, j_first, piece_first, pieces_first, c_first_first);
      pieces_of(p, u_last, 0, piece_last, pieces_last, c_first_last);
    } else {
      u = blockIdx.x;
      item = 0;
      items = u < p.num_units ? unit_items(p, u) : 0;
    }
  }
  // Number of CTAs c >= 1 whose step range begins at or before step x.
  __device__ __forceinline__ static long long starts_le(const FwdParams& p, long long x) {
    const long long g = gridDim.x;
    const long long c = ((x + 1) * g - 1) / p.total_steps;
    return c < g - 1 ? c : g - 1;
  }
  // Piece index of the part of unit uu starting at key tile j0, the unit's
  // number of pieces, and the CTA holding piece 0.
  __device__ __forceinline__ static void pieces_of(const FwdParams& p, int uu, int j0, int& piece,
                                                   int& pieces, int& c_first) {
    const int steps = split_unit_steps(p, uu % p.num_q_pairs);
    const long long a = split_unit_start(p, uu);
    const long long ca = starts_le(p, a);
    piece = static_cast<int>(starts_le(p, a + j0) - ca);
    pieces = static_cast<int>(1 + starts_le(p, a + steps - 1) - ca);
    c_first = static_cast<int>(ca);
  }
  __device__ __forceinline__ bool next(const FwdParams& p, Unit& w) {
    if constexpr (SPLIT) {
      if (u > u_last) return false;
      const bool first = (item == 0);
      const int j0 = first ? j_first : 0;
      const int j1 = (u == u_last) ? j_end : split_unit_steps(p, u % p.num_q_pairs);
      w = decode_item<false, true>(p, u, 0);
      w.jbase = j0;
      // key tiles [j0, j1) of the unit; a query tile sees only those below
      // its own count (under the causal mask the first tile of a pair sees
      // one fewer than the second, and may see none of a late piece)
      w.n[0] = max(0, min(j1, w.n[0]) - j0);
      w.n[1] = max(0, min(j1, w.n[1]) - j0);
      w.nmax = max(w.n[0], w.n[1]);
      if (first) {
        w.piece = piece_first;
        w.pieces = pieces_first;
        w.c_first = c_first_first;
      } else if (u == u_last) {
        w.piece = piece_last;
        w.pieces = pieces_last;
        w.c_first = c_first_last;
      } else {
        w.piece = 0;
        w.pieces = 1;
        w.c_first = static_cast<int>(blockIdx.x);
      }
      item = 1;
      ++u;
      return true;
    } else {
      while (item >= items) {
        u += gridDim.x;
        if (u >= p.num_units) return false;
        item = 0;
        items = unit_items(p, u);
      }
      w = decode_item<DUAL>(p, u, item++);
      return true;
    }
  }
};

// Piece k of a split unit lives in CTA (c_first + k): piece 0 is that CTA's
// last item (it runs to the end of the CTA's range), every later piece is
// its CTA's first item (it starts the range), so one CTA holds at most one
// piece in each of its two workspace slots.
__device__ __forceinline__ size_t ws_row(int cta, int slot, int t, int r) {
  return ((static_cast<size_t>(cta) * 2 + slot) * 2 + t) * BLOCK_M + r;
}
// A slot's O is stored column-major (column c of row r at c * 128 + r), so
// the 32 rows of a warp read and write 32 consecutive floats.
__device__ __forceinline__ size_t ws_o_base(int cta, int slot, int t, int D) {
  return ((static_cast<size_t>(cta) * 2 + slot) * 2 + t) * static_cast<size_t>(BLOCK_M) * D;
}


// The S sequence of one item: the MMA warp computes the score tiles of the
// two Q tiles alternately, S_0(0), S_1(0), S_0(1), S_1(1), ..., and, when
// one tile visits one more K/V tile than the other, the longer tile's last
// one at the end.  Position k of that sequence goes to S/P buffer
// (k_item_base + k) % NSB.
struct SeqPos {
  int t, j;
};
__device__ __forceinline__ SeqPos seq_at(const Unit& w, int k) {
  const int m = min(w.n[0], w.n[1]);
  if (k < 2 * m) return {k & 1, k >> 1};
  return {w.n[0] > w.n[1] ? 0 : 1, m + (k - 2 * m)};
}
__device__ __forceinline__ int seq_pos(const Unit& w, int t, int j) {
  const int m = min(w.n[0], w.n[1]);
  return j < m ? 2 * j + t : 2 * m + (j - m);
}
// Ring slot (counted from the item's first) of the K or V tile that score
// tile (t, j) uses: one per key step, or one per tile in a dual unit.
template <bool DUAL>
__device__ __forceinline__ int kv_slot(const Unit& w, SeqPos s) {
  return (DUAL && w.kvs == 2) ? 2 * s.j + s.t : s.j;
}
// That K / V tile is used for the last time by tile 1, by tile 0 when tile 1
// does not visit j, and always in a dual unit (each tile has its own).
template <bool DUAL>
__device__ __forceinline__ bool last_use(const Unit& w, SeqPos s) {
  return (DUAL && w.kvs == 2) || s.t == 1 || s.j >= w.n[1];
}

// P for one 128-key row: p = 2^(s * sl2 + neg_m), packed two keys per word
// (even key low; e4m3: four keys per word, lowest key in the low byte), and
// the fp32 sum of the unrounded values.  Of every 16 key pairs,
// exp_poly_pairs<D, FP8>() take 2^x from the FMA-pipe polynomial.
// d = 64 and e4m3 operands (both bound by the softmax) try the running max
// as it stands before computing a row max; at d = 128 with 16-bit operands
// the extra registers of that path cost more than it saves (e4m3 P needs
// half the packed registers, 32 words per row).
template <int D, bool FP8 = false>
__host__ __device__ constexpr bool kStaleMaxFirst() { return D == 64 || FP8; }

// With the running max as it stands (STALE) x has no upper bound.  The
// MUFU's 2^x overflows to +inf for x >= 128, which the caller's sum check
// rejects, but the polynomial's exponent add wraps past x = 128 into small or
// negative values that the sum would not reveal.  So a STALE call also
// returns the largest x given to the polynomial, and the caller accepts the
// row only if it stays below POLY_X_LIMIT, where the polynomial is exact to
// its stated error (every x >= 15 then gives a P >= 2^15, which the sum
// check rejects).  Without STALE, x <= RESCALE_LOG2 by construction.
constexpr float POLY_X_LIMIT = 64.0f;

template <int D, bool BF16, bool STALE, bool FP8 = false>
__device__ __forceinline__ float exp_row(const float (&s)[128], float sl2, float neg_m,
                                         uint32_t (&pk)[FP8 ? 32 : 64], float& xp_max) {
  float sum0 = 0.f, sum1 = 0.f;
  float xm = -INFINITY;
  float prev0 = 0.f, prev1 = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    float x0, x1, a, bb;
    fma2(x0, x1, s[2 * i], s[2 * i + 1], sl2, sl2, neg_m, neg_m);
    if (i % 16 < exp_poly_pairs<D, FP8>()) {
      if constexpr (STALE) xm = max3(xm, x0, x1);
      exp2_poly2(a, bb, x0, x1);  // FMA pipe, in parallel with the MUFU ones
    } else {
      a = ex2_approx(x0);
      bb = ex2_approx(x1);
    }
    add2(sum0, sum1, sum0, sum1, a, bb);
    if constexpr (FP8) {
      if (i % 2 == 0) {
        prev0 = a;
        prev1 = bb;
      } else {
        pk[i / 2] = pack4_e4m3(prev0, prev1, a, bb);
      }
    } else {
      pk[i] = pack2<BF16>(a, bb);
    }
  }
  xp_max = xm;
  return sum0 + sum1;
}

// Bounded wait until the 32-bit shared-memory counter at `addr` reaches
// `target` (acquire load; same time limit and abort handling as wait_phase).
__device__ __forceinline__ bool wait_count(uint32_t addr, uint32_t target, volatile int* abort_flag,
                                           uint32_t site) {
  uint32_t spins = 0;
  uint64_t t0 = 0;
  while (ld_acquire_shared(addr) < target) {
    if ((++spins & 1023u) == 0) {
      const uint64_t now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > WAIT_LIMIT_NS) {
        atomicCAS(&g_attn_status, 0u, 0x80000000u | site);
        *abort_flag = 1;
        return false;
      }
      if (*abort_flag) return false;
    }
  }
  return true;
}

// Bounded wait on one mbarrier phase, fully inlined (a call here would make
// the compiler save live registers to local memory on every slow wait).
// Returns false on timeout (status word set, abort flag raised) or, when
// honour_abort, once another role has aborted.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint32_t site, bool honour_abort = true) {
  // a phase that has already completed is found by the non-blocking test;
  // only an open phase enters the (suspending) try_wait loop
  if (mbar_test_wait(bar, parity)) return true;
  uint32_t spins = 0;
  uint64_t t0 = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++spins & 1023u) == 0) {
      const uint64_t now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > WAIT_LIMIT_NS) {
        atomicCAS(&g_attn_status, 0u, 0x80000000u | site);
        *abort_flag = 1;
        return false;
      }
      if (honour_abort && *abort_flag) return false;
    }
  }
  return true;
}

// DUAL: the unit-mode kernel for problems with dual units (an odd number of
// query tiles per head); the other unit-mode problems run the DUAL = false
// instantiation, which carries none of the dual-unit bookkeeping.
// FP8: Q, K and Vt are e4m3 (tm_v then maps Vt [B H, d, Nk]); O is written as
// bf16 (BF16 must be true).
template <int D, bool BF16, bool SPLIT, bool DUAL, bool FP8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(!FP8 || (D == 128 && BF16), "e4m3 operands: d = 128, bf16 output");
  using L = SmemLayout<D, FP8>;
  constexpr int NSB = L::NSB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  auto bar = [&](int i) -> uint32_t { return sbase + L::BAR_OFF + 8u * i; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::K_STAGES; ++s) {
      mbar_init(bar(L::K_FULL + s), 1);
      mbar_init(bar(L::K_EMPTY + s), 1);
    }
    for (int s = 0; s < L::V_STAGES; ++s) {
      mbar_init(bar(L::V_FULL + s), 1);
      mbar_init(bar(L::V_EMPTY + s), 1);
    }
    for (int s = 0; s < L::Q_SLOTS; ++s) {
      mbar_init(bar(L::Q_FULL + s), 1);
      mbar_init(bar(L::Q_EMPTY + s), 1);
    }
    for (int b = 0; b < NSB; ++b) {
      mbar_init(bar(L::S_FULL + 2 * b), 1);
      mbar_init(bar(L::S_FULL + 2 * b + 1), 1);
      mbar_init(bar(L::P_FULL + b), 4 * 32);
    }
    mbar_init(bar(L::O_READY + 0), 1);
    mbar_init(bar(L::O_READY + 1), 1);
    for (int b = 0; b < NSB; ++b) mbar_init(bar(L::PV_DONE + b), 1);
    mbar_init(bar(L::DRAIN + 0), 1);
    mbar_init(bar(L::DRAIN + 1), 1);
    mbar_init(bar(L::SYNC), 2 * 128);
    mbar_init(bar(L::NEVER), 1);
    *abort_flag = 0;
    reinterpret_cast<uint32_t*>(smem + L::PV_DONE_OFF)[0] = 0u;
    reinterpret_cast<uint32_t*>(smem + L::PV_DONE_OFF)[1] = 0u;
    fence_mbarrier_init();
  }
  if (warp == LOAD_WARP && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
  }
  if (warp == VLOAD_WARP && lane == 0) prefetch_tensormap(&tm_v);
  if (warp == MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp >= 8) {
    regs_decrease<producer_regs<SPLIT>()>();
    // The producer warps run their loops on all 32 lanes, so every address,
    // coordinate and descriptor is warp-uniform and stays in uniform
    // registers; one elected lane issues the TMA and tcgen05 instructions
    // (a loop on one lane would have to move each operand into uniform
    // registers before every MMA, which made the issue the bottleneck).
    const bool leader = elect_one();
    const uint32_t q_smem = sbase + L::Q_OFF;
    const uint32_t k_smem = sbase + L::K_OFF;
    const uint32_t v_smem = sbase + L::V_OFF;
    auto warp_wait = [&](uint32_t b, uint32_t parity, uint32_t site) -> bool {
      const bool r = wait_phase(b, parity, abort_flag, site);
      return __all_sync(0xffffffffu, r);
    };
    if (warp == LOAD_WARP || warp == VLOAD_WARP) {
      // ----------------------------------------------------------- TMA producers
      // Warp 9 loads each item's two Q tiles and K_0..K_{n-1}; warp 11 loads
      // V_0..V_{n-1}.  Each ring is consumed in increasing j, so each loader
      // streams its ring in that order and neither waits behind the other's
      // free slots.
      const bool is_k = (warp == LOAD_WARP);
      const int stages = is_k ? L::K_STAGES : L::V_STAGES;
      const uint32_t ring = is_k ? k_smem : v_smem;
      const int full0 = is_k ? L::K_FULL : L::V_FULL;
      const int empty0 = is_k ? L::K_EMPTY : L::V_EMPTY;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint32_t pos = 0, items_done = 0;
      bool ok = true;
      WorkCursor<SPLIT, DUAL> cur(p);
      Unit w;
      while (ok && cur.next(p, w)) {
        {
          if (is_k) {
            if (p.stall_site == STALL_LOAD) {
              warp_wait(bar(L::NEVER), 0, SITE_INJECTED);
              ok = false;
              break;
            }
            // item i uses Q slot i % Q_SLOTS, free again once the S MMAs of
            // item i - Q_SLOTS have completed
            const uint32_t qs = items_done % L::Q_SLOTS;
            if (items_done >= static_cast<uint32_t>(L::Q_SLOTS)) {
              ok = warp_wait(bar(L::Q_EMPTY + qs), (items_done / L::Q_SLOTS - 1) & 1,
                             SITE_LOAD_Q_EMPTY);
              if (!ok) break;
            }
            if (leader) {
              mbar_arrive_expect_tx(bar(L::Q_FULL + qs), 2 * L::TILE_BYTES);
#pragma unroll
              for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int h = 0; h < L::HALVES; ++h)
                  tma_load_3d(q_smem + (2 * qs + t) * L::TILE_BYTES + h * L::HALF_BYTES, &tm_q,
                              bar(L::Q_FULL + qs), h * 64,
                              (DUAL && t) ? w.q1 : w.q0 + t * BLOCK_M, (DUAL && t) ? w.bh1 : w.bh);
            }
            __syncwarp();
          }
          ++items_done;
          const int kvs = DUAL ? w.kvs : 1;
          for (int x = 0; ok && x < w.nmax * kvs; ++x) {
            const int j = (DUAL && kvs == 2) ? x / 2 : x;
            const int bh = (DUAL && kvs == 2 && (x & 1)) ? w.bh1 : w.bh;
            const uint32_t st = pos % stages, ph = (pos / stages) & 1;
            if (pos >= static_cast<uint32_t>(stages) &&
                !warp_wait(bar(empty0 + st), ph ^ 1, SITE_LOAD_KV_EMPTY)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_arrive_expect_tx(bar(full0 + st), L::TILE_BYTES);
              if (FP8 && !is_k) {  // Vt tile: all d rows, keys (jbase + j) * 128 ..
                tma_load_3d(ring + st * L::TILE_BYTES, map, bar(full0 + st),
                            (w.jbase + j) * BLOCK_N, 0, bh);
              } else {
#pragma unroll
                for (int h = 0; h < L::HALVES; ++h)
                  tma_load_3d(ring + st * L::TILE_BYTES + h * L::HALF_BYTES, map, bar(full0 + st),
                              h * 64, (w.jbase + j) * BLOCK_N, bh);
              }
            }
            __syncwarp();
            ++pos;
          }
        }
      }
      // Every issued load must have landed before the CTA may exit.
      for (uint32_t i = pos > static_cast<uint32_t>(stages) ? pos - stages : 0; i < pos; ++i)
        wait_phase(bar(full0 + i % stages), (i / stages) & 1, abort_flag, SITE_DRAIN, false);
      if (is_k) {
        for (uint32_t i = items_done > static_cast<uint32_t>(L::Q_SLOTS) ? items_done - L::Q_SLOTS : 0;
             i < items_done; ++i)
          wait_phase(bar(L::Q_FULL + i % L::Q_SLOTS), (i / L::Q_SLOTS) & 1, abort_flag, SITE_DRAIN,
                     false);
      }
      __syncwarp();
    } else if (warp == MMA_WARP || warp == PV_WARP) {
      // ----------------------------------------------------------- MMA issuers
      // Two warps feed the tensor core.  Warp 8 issues S(g) = Q_t K_j^T for
      // the g-th score tile of the CTA into S/P buffer g % NSB as soon as
      // its K tile is loaded and the P V that last read that buffer is done;
      // it can therefore run up to NSB tiles ahead of the softmax.  Warp 10
      // issues O_t += P(g) V_j as soon as the softmax has written P(g).  Each
      // warp only waits on its own inputs, so one waiting for the softmax
      // does not hold back the other's work.
      constexpr uint32_t IDESC_S =
          FP8 ? idesc_e4m3(BLOCK_M, BLOCK_N) : idesc_f16(BF16, false, false, BLOCK_M, BLOCK_N);
      constexpr uint32_t IDESC_O = FP8 ? idesc_e4m3(BLOCK_M, D) : idesc_f16(BF16, false, true, BLOCK_M, D);
      // S: both operands K-major (head dim contiguous), 128-byte swizzle,
      // 8-row groups 1024 bytes apart; each k-step covers 16 elements = 32
      // bytes of a 128-byte row, the head dim > 64 continues in the next 16 KB
      // slab.  Descriptors are built once; a k-step or a ring slot only adds
      // (byte offset >> 4) to the start-address field (every address stays
      // below 256 KB, so the add never carries out of it).
      const uint64_t q_desc = sw128_desc(q_smem, 16, 1024);
      const uint64_t k_desc = sw128_desc(k_smem, 16, 1024);
      // P V: P from TMEM (16 keys = 8 columns per k-step), V MN-major (head
      // dim contiguous): 8-key groups 1024 bytes apart, 64-column slabs 16 KB
      // apart; each k-step advances 16 keys = 2 KB.  e4m3: S and P V both take
      // 32 elements = 32 bytes per k-step; P from TMEM (32 keys = 8 columns),
      // Vt K-major like K (keys contiguous, d rows in 8-row groups 1 KB apart).
      const uint64_t v_desc =
          FP8 ? sw128_desc(v_smem, 16, 1024) : sw128_desc(v_smem, L::HALF_BYTES, 1024);
      const uint32_t tmem_s = tmem_base + L::S_COL;
      const uint32_t tmem_o = tmem_base + L::O_COL;
      // With only two S/P buffers (d = 128) the next S of a tile must reuse
      // the buffer its last P V reads; one thread issuing both keeps them in
      // order in the tensor pipe without waiting for the P V to finish, so
      // at d = 128 warp 8 issues everything in sequence order (P V(g), then
      // S(g + 2)) and warp 10 idles.
      constexpr bool kSplit = (NSB > 2);
      if (!kSplit && warp == PV_WARP) {
        // nothing to do
      } else {
      const bool is_s = (warp == MMA_WARP);

      uint32_t pos = 0, g = 0;  // ring position of K_0 / V_0 of the item; score tile count
      uint32_t items = 0;       // items begun (the Q slot is items % Q_SLOTS)
      uint32_t buf = 0, round = 0;           // g % NSB, g / NSB
      uint32_t pv_ph0 = 0, pv_ph1 = 0, pv_n0 = 0, pv_n1 = 0;  // P V issuer: O_READY phases, counts
      bool ok = true;
      WorkCursor<SPLIT, DUAL> cur(p);
      Unit w;
      while (ok && cur.next(p, w)) {
        {
          const int total = w.n[0] + w.n[1];
          if (is_s) {
            if (p.stall_site == STALL_MMA) {
              warp_wait(bar(L::NEVER), 0, SITE_INJECTED);
              ok = false;
              break;
            }
            ok = warp_wait(bar(L::Q_FULL + items % L::Q_SLOTS), (items / L::Q_SLOTS) & 1,
                           SITE_MMA_Q_FULL);
            if (!ok) break;
          }
          const uint32_t q_slot = items % L::Q_SLOTS;
          const uint64_t q_item = q_desc + q_slot * static_cast<uint32_t>((2 * L::TILE_BYTES) >> 4);
          int ready_j = -1;
          if constexpr (!kSplit) {
            // in-order issue: S(0), S(1), then P V(k) followed by S(k + 2)
            int k_ready = -1, v_ready = -1;
            auto issue_s = [&](int k) -> bool {
              const SeqPos sp = seq_at(w, k);
              const int slot = kv_slot<DUAL>(w, sp);
              const uint32_t kp = pos + slot;
              const uint32_t st = kp % L::K_STAGES;
              if (slot > k_ready) {
                if (!warp_wait(bar(L::K_FULL + st), (kp / L::K_STAGES) & 1, SITE_MMA_KV_FULL))
                  return false;
                tc_fence_after();
                k_ready = slot;
              }
              const uint32_t b = (g + k) % NSB;
              const uint64_t a = q_item + static_cast<uint32_t>(sp.t * (L::TILE_BYTES >> 4));
              const uint64_t bd = k_desc + st * static_cast<uint32_t>(L::TILE_BYTES >> 4);
              if (leader) {
                if constexpr (FP8) {
#pragma unroll
                  for (int kk = 0; kk < D / 32; ++kk)
                    mma_ss_f8(tmem_s + 128 * b, a + kk * 2, bd + kk * 2, IDESC_S, kk > 0 ? 1u : 0u);
                } else {
#pragma unroll
                  for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk / 4) * L::HALF_BYTES + (kk % 4) * 32) >> 4;
                    mma_ss(tmem_s + 128 * b, a + off, bd + off, IDESC_S, kk > 0 ? 1u : 0u);
                  }
                }
                mma_commit(bar(L::S_FULL + 2 * b + sp.t));
                if (last_use<DUAL>(w, sp)) mma_commit(bar(L::K_EMPTY + st));
              }
              return true;
            };
            for (int k = 0; ok && k < min(NSB, total); ++k) ok = issue_s(k);
            for (int k = 0; ok && k < total; ++k) {
              const SeqPos sp = seq_at(w, k);
              const int slot = kv_slot<DUAL>(w, sp);
              const uint32_t vp = pos + slot;
              const uint32_t st = vp % L::V_STAGES;
              if (slot > v_ready) {
                if (!warp_wait(bar(L::V_FULL + st), (vp / L::V_STAGES) & 1, SITE_MMA_KV_FULL)) {
                  ok = false;
                  break;
                }
                v_ready = slot;
              }
              const uint32_t gk = g + k;
              const uint32_t b = gk % NSB;
              if (!warp_wait(bar(L::P_FULL + b), (gk / NSB) & 1, SITE_MMA_P_FULL)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t bd = v_desc + st * static_cast<uint32_t>(L::TILE_BYTES >> 4);
              if (leader) {
                if constexpr (FP8) {
#pragma unroll
                  for (int kk = 0; kk < BLOCK_N / 32; ++kk)
                    mma_ts_f8(tmem_o + D * sp.t, tmem_s + 128 * b + kk * 8, bd + kk * 2, IDESC_O,
                              (sp.j > 0 || kk > 0) ? 1u : 0u);
                } else {
#pragma unroll
                  for (int kk = 0; kk < BLOCK_N / 16; ++kk)
                    mma_ts(tmem_o + D * sp.t, tmem_s + 128 * b + kk * 8, bd + kk * (2048 >> 4),
                           IDESC_O, (sp.j > 0 || kk > 0) ? 1u : 0u);
                }
                // in-order issue: S_t(j + 1) completing already implies this
                // P V completed, so only the tile's last P V is signalled
                if (sp.j + 1 == (sp.t ? w.n[1] : w.n[0])) mma_commit(bar(L::O_READY + sp.t));
                if (last_use<DUAL>(w, sp)) mma_commit(bar(L::V_EMPTY + st));
              }
              // the buffer of P(k) is refilled by S(k + NSB): same thread, so
              // the tensor pipe runs it after this P V
              if (k + NSB < total) ok = issue_s(k + NSB);
            }
            g += total;
          } else
          for (int k = 0; k < total; ++k) {
            const SeqPos sp = seq_at(w, k);
            const int slot = kv_slot<DUAL>(w, sp);
            if (is_s) {
              const uint32_t kp = pos + slot;
              const uint32_t st = kp % L::K_STAGES;
              if (slot > ready_j) {
                if (!warp_wait(bar(L::K_FULL + st), (kp / L::K_STAGES) & 1, SITE_MMA_KV_FULL)) {
                  ok = false;
                  break;
                }
                ready_j = slot;
              }
              if (g >= static_cast<uint32_t>(NSB) &&
                  !warp_wait(bar(L::PV_DONE + buf), (round - 1) & 1, SITE_MMA_P_FULL)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t a = q_item + static_cast<uint32_t>(sp.t * (L::TILE_BYTES >> 4));
              const uint64_t bd = k_desc + st * static_cast<uint32_t>(L::TILE_BYTES >> 4);
              if (leader) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                  const uint32_t off = ((kk / 4) * L::HALF_BYTES + (kk % 4) * 32) >> 4;
                  mma_ss(tmem_s + 128 * buf, a + off, bd + off, IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(L::S_FULL + 2 * buf + sp.t));
                if (last_use<DUAL>(w, sp)) mma_commit(bar(L::K_EMPTY + st));
              }
            } else {
              const uint32_t vp = pos + slot;
              const uint32_t st = vp % L::V_STAGES;
              if (slot > ready_j) {
                if (!warp_wait(bar(L::V_FULL + st), (vp / L::V_STAGES) & 1, SITE_MMA_KV_FULL)) {
                  ok = false;
                  break;
                }
                ready_j = slot;
              }
              if (!warp_wait(bar(L::P_FULL + buf), round & 1, SITE_MMA_P_FULL)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t bd = v_desc + st * static_cast<uint32_t>(L::TILE_BYTES >> 4);
              if (leader) {
#pragma unroll
                for (int kk = 0; kk < BLOCK_N / 16; ++kk)
                  mma_ts(tmem_o + D * sp.t, tmem_s + 128 * buf + kk * 8, bd + kk * (2048 >> 4),
                         IDESC_O, (sp.j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar(L::O_READY + sp.t));
                mma_commit(bar(L::PV_DONE + buf));
                if (last_use<DUAL>(w, sp)) mma_commit(bar(L::V_EMPTY + st));
              }
              // Wait for this P V and publish the tile's completed count: the
              // softmax reads O (to rescale it or in the epilogue) only once the
              // count covers every P it has handed over.  The next P V waits for
              // the other tile's P anyway, so this wait costs the issue nothing.
              {
                const uint32_t ph = sp.t ? pv_ph1 : pv_ph0;
                if (!warp_wait(bar(L::O_READY + sp.t), ph, SITE_MMA_P_FULL)) {
                  ok = false;
                  break;
                }
                if (sp.t) { pv_ph1 ^= 1u; ++pv_n1; } else { pv_ph0 ^= 1u; ++pv_n0; }
                tc_fence_before();
                if (leader)
                  st_release_shared(smem_addr(smem + L::PV_DONE_OFF) + 4 * sp.t, sp.t ? pv_n1 : pv_n0);
              }
            }
            ++g;
            if (++buf == static_cast<uint32_t>(NSB)) {
              buf = 0;
              ++round;
            }
          }
          if (!ok) break;
          // every S of the item has been issued: the Q tiles may be replaced
          // once those MMAs complete
          if (is_s && leader) mma_commit(bar(L::Q_EMPTY + q_slot));
          ++items;
          __syncwarp();
          pos += DUAL ? w.nmax * w.kvs : w.nmax;
        }
      }
      // All MMAs (and their commits) must be finished before TMEM is freed.
      const uint32_t drain = bar(L::DRAIN + (is_s ? 0 : 1));
      if (leader) mma_commit(drain);
      __syncwarp();
      wait_phase(drain, 0, abort_flag, SITE_DRAIN, false);
      __syncwarp();
      }
    }
  } else {
    regs_increase<softmax_regs<SPLIT>()>();
    // ------------------------------------------------------------- softmax
    const int t = warp / 4;
    const int quarter = warp % 4;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS0 = tmem_base + lane_off + L::S_COL;
    const uint32_t tO = tmem_base + lane_off + L::O_COL + D * t;
    const float sl2 = p.scale_log2;
    uint32_t o_phase = 0, sk = 0;
    uint32_t pv_handed = 0;  // P tiles of this Q tile handed to the P V MMA so far
    uint32_t s_parity = 0;  // bit b: parity of the next S_FULL(b, t) phase this warpgroup waits for
    bool ok = true;
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
    uint32_t sync_phase = 0;
    auto softmax_sync = [&]() -> bool {
      mbar_arrive(bar(L::SYNC));
      const bool r = wait_phase(bar(L::SYNC), sync_phase, abort_flag, SITE_SOFTMAX_SYNC);
      sync_phase ^= 1;
      return __all_sync(0xffffffffu, r);
    };
    WorkCursor<SPLIT, DUAL> cur(p);
    Unit w;
    while (ok && cur.next(p, w)) {
      {
        const int n = t ? w.n[1] : w.n[0];
        const uint32_t item_sk = sk;
        sk += w.n[0] + w.n[1];
        if (n == 0 && (!SPLIT || w.pieces == 1)) continue;
        const int q_start = (DUAL && t) ? w.q1 : w.q0 + t * BLOCK_M;
        const int bh = (DUAL && t) ? w.bh1 : w.bh;
        const int row = q_start + r;
        // last key this row may see (top-left causal: key j <= query i)
        const int last_key = p.causal ? min(p.Nk - 1, row) : (p.Nk - 1);
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < n; ++j) {
          const uint32_t kg = item_sk + seq_pos(w, t, j);
          const uint32_t b = kg % NSB;
          const uint32_t tS = tS0 + 128 * b;
          if (p.stall_site == STALL_SOFTMAX && t == 0) {
            wait_phase(bar(L::NEVER), 0, abort_flag, SITE_INJECTED);
            ok = false;
            break;
          }
          ok = wait_phase(bar(L::S_FULL + 2 * b + t), (s_parity >> b) & 1u, abort_flag,
                          SITE_SOFTMAX_S_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          s_parity ^= 1u << b;
          tc_fence_after();
          bool raise = false;
          float alpha = 1.f, m_new = m;
          if constexpr (kStaleMaxFirst<D, FP8>()) {
            // S of this tile, keys past the row's last visible key set to -inf
            float s[128];
            auto load_s = [&]() {
              uint32_t sr[128];
#pragma unroll
              for (int c = 0; c < 4; ++c)
                tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * c));
              tmem_wait_ld_regs(sr);
#pragma unroll
              for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
              const int k0 = (w.jbase + j) * BLOCK_N;
              const bool need_mask = (k0 + BLOCK_N > p.Nk) || (p.causal && k0 + BLOCK_N - 1 > q_start);
              if (need_mask) {
                const int lim = last_key - k0;  // columns > lim are masked
#pragma unroll
                for (int c = 0; c < 128; ++c) s[c] = (c > lim) ? -INFINITY : s[c];
              }
            };
            load_s();

            // P = 2^(s * scale * log2 e - m), packed two keys per 32-bit word
            // (even key in the low half; e4m3: four per word).  After the
            // first tile the running max m is tried as it stands: the sum of
            // the tile's P bounds every P, so if it stays below 2^15 (e4m3:
            // 448, its largest finite value) and every exponent given to the
            // polynomial lies in its valid range (see exp_row), no P overflows
            // its format and the result is exact with the stale max, and the
            // row max is never computed.  Otherwise (or on the first
            // tile) S is read again and the row max decides, as below.  P is
            // written to TMEM only after that decision, so S is still there
            // to be read again.
            uint32_t pk[FP8 ? 32 : 64];
            float tsum = 0.f;
            bool settled = false;
            if (j > 0) {
              float xp_max;
              tsum = exp_row<D, BF16, true, FP8>(s, sl2, -m, pk, xp_max);
              // every P below the largest finite value of its format
              settled = __all_sync(0xffffffffu,
                                   tsum < (FP8 ? 448.f : 32768.f) && xp_max < POLY_X_LIMIT);
              if (!settled) load_s();
            }
            if (!settled) {
              // row max: eight independent chains of three-input max over s[0..127]
              float mx[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) mx[i] = max3(s[2 * i], s[2 * i + 1], s[16 + 2 * i]);
#pragma unroll
              for (int c = 32; c < 128; c += 16) {
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
              }
#pragma unroll
              for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[17 + 2 * i]);
              const float mx_all = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]),
                                        fmaxf(mx[6], mx[7]));
              // The running max only moves when the tile raises it by more than
              // RESCALE_LOG2 (base 2): until then exponents stay below
              // 2^RESCALE_LOG2 and O, l and lse keep using the same stale max,
              // so the result is unchanged while most O rescales are skipped.
              const float m_cand = fmaxf(m, mx_all * sl2);
              raise = m_cand > m + RESCALE_LOG2;
              m_new = raise ? m_cand : m;
              const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
              alpha = raise ? ex2_approx(m - m_use) : 1.f;
              float xp_unused;
              tsum = exp_row<D, BF16, false, FP8>(s, sl2, -m_use, pk, xp_unused);
            }
            tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(pk));
            if constexpr (!FP8) tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
            l = l * alpha + tsum;
            m = m_new;
          } else {
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(sr + 32 * c));
            tmem_wait_ld_regs(sr);
            float s[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);

            const int k0 = (w.jbase + j) * BLOCK_N;
            const bool need_mask = (k0 + BLOCK_N > p.Nk) || (p.causal && k0 + BLOCK_N - 1 > q_start);
            if (need_mask) {
              const int lim = last_key - k0;  // columns > lim are masked
#pragma unroll
              for (int c = 0; c < 128; ++c) s[c] = (c > lim) ? -INFINITY : s[c];
            }
            // row max: eight independent chains of three-input max over s[0..127]
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = max3(s[2 * i], s[2 * i + 1], s[16 + 2 * i]);
#pragma unroll
            for (int c = 32; c < 128; c += 16) {
#pragma unroll
              for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[17 + 2 * i]);
            const float mx_all = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]),
                                      fmaxf(mx[6], mx[7]));
            // The running max only moves when the tile raises it by more than
            // RESCALE_LOG2 (base 2): until then exponents stay below
            // 2^RESCALE_LOG2 and O, l and lse keep using the same stale max, so
            // the result is unchanged while most O rescales are skipped.
            const float m_cand = fmaxf(m, mx_all * sl2);
            raise = m_cand > m + RESCALE_LOG2;
            m_new = raise ? m_cand : m;
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            alpha = raise ? ex2_approx(m - m_use) : 1.f;
            const float neg_m = -m_use;

            // P = 2^(s * scale * log2 e - m), packed two keys per 32-bit TMEM
            // column (even key in the low half), written over S in 16-column
            // chunks so each chunk's S registers die as it is stored.  e4m3:
            // four keys per column (lowest key in the low byte), 8-column
            // chunks; P < 2^RESCALE_LOG2 = 256 stays inside e4m3's range.
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int chunk = 0; chunk < 4; ++chunk) {
              if constexpr (FP8) {
                uint32_t pk[8];
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                  float e[4];
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const int c = 2 * c4 + h;  // key pair within the chunk
                    float x0, x1;
                    fma2(x0, x1, s[32 * chunk + 2 * c], s[32 * chunk + 2 * c + 1], sl2, sl2, neg_m,
                         neg_m);
                    if (c < exp_poly_pairs<D, FP8>()) {
                      exp2_poly2(e[2 * h], e[2 * h + 1], x0, x1);
                    } else {
                      e[2 * h] = ex2_approx(x0);
                      e[2 * h + 1] = ex2_approx(x1);
                    }
                    add2(sum0, sum1, sum0, sum1, e[2 * h], e[2 * h + 1]);
                  }
                  pk[c4] = pack4_e4m3(e[0], e[1], e[2], e[3]);
                }
                tmem_st8(tS + 8 * chunk, pk);
                continue;
              }
              uint32_t pk[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                float x0, x1, a, bb;
                fma2(x0, x1, s[32 * chunk + 2 * c], s[32 * chunk + 2 * c + 1], sl2, sl2, neg_m, neg_m);
                if (c < exp_poly_pairs<D>()) {
                  exp2_poly2(a, bb, x0, x1);  // FMA pipe, in parallel with the MUFU ones
                } else {
                  a = ex2_approx(x0);
                  bb = ex2_approx(x1);
                }
                add2(sum0, sum1, sum0, sum1, a, bb);
                pk[c] = pack2<BF16>(a, bb);
              }
              tmem_st16(tS + 16 * chunk, pk);
            }
            l = l * alpha + (sum0 + sum1);
            m = m_new;
          }

          // O_t may only be touched once the previous P V of this tile is
          // done: with split issue that is its own signal; with in-order issue
          // (two S buffers) the S just read was queued behind that P V.
          if (j > 0 && __any_sync(0xffffffffu, raise)) {
            if constexpr (NSB > 2) {
              ok = wait_count(smem_addr(smem + L::PV_DONE_OFF) + 4 * t, pv_handed, abort_flag,
                              SITE_SOFTMAX_O_READY);
              ok = __all_sync(0xffffffffu, ok);
              if (!ok) break;
              tc_fence_after();
            }
            {
#pragma unroll
              for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tO + c0, o);
                tmem_wait_ld_regs(o);
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                  float a0, a1;
                  mul2(a0, a1, __uint_as_float(o[i]), __uint_as_float(o[i + 1]), alpha, alpha);
                  o[i] = __float_as_uint(a0);
                  o[i + 1] = __float_as_uint(a1);
                }
                tmem_st32(tO + c0, o);
              }
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(L::P_FULL + b));
          ++pv_handed;
        }
        if (!ok) break;

        // --------------------------------------------------------- epilogue
        const bool in_range = row < p.Nq;
        // this piece's statistics, for the merge; a piece in which this query
        // tile sees no key (under the causal mask) has lse = -inf, weight 0
        float lse_self = -INFINITY, inv_self = 0.f;
        if (n > 0) {
          if constexpr (NSB > 2) {
            ok = wait_count(smem_addr(smem + L::PV_DONE_OFF) + 4 * t, pv_handed, abort_flag,
                            SITE_SOFTMAX_O_READY);
          } else {
            ok = wait_phase(bar(L::O_READY + t), o_phase, abort_flag, SITE_SOFTMAX_O_READY);
            o_phase ^= 1;
          }
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float inv_l = (FP8 ? p.o_scale : 1.f) / l;
          const float lse_row = (m + lg2_approx(l)) * 0.69314718055994531f;
          lse_self = lse_row;
          inv_self = inv_l;
          if (!SPLIT || w.pieces == 1) {
            uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) +
                                                   (static_cast<size_t>(bh) * p.Nq + row) * D);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c0, o);
              tmem_wait_ld_regs(o);
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l,
                                    __uint_as_float(o[2 * i + 1]) * inv_l);
              if (in_range) {
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                  orow[c0 / 8 + v4] =
                      make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
              }
            }
            if (p.lse != nullptr && in_range)
              p.lse[static_cast<size_t>(bh) * p.Nq + row] = lse_row;
          } else {
            // a piece of a split unit: normalised O and lse to this CTA's slot
            const int slot = w.piece == 0 ? 1 : 0;
            const size_t wr = ws_row(blockIdx.x, slot, t, r);
            float* so = p.ws_o + ws_o_base(blockIdx.x, slot, t, D) + r;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c0, o);
              tmem_wait_ld_regs(o);
              if (in_range) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  __stcg(so + static_cast<size_t>(c0 + c) * BLOCK_M, __uint_as_float(o[c]) * inv_l);
              }
            }
            if (in_range) __stcg(p.ws_lse + wr, lse_row);
          }
          tc_fence_before();
        } else if (SPLIT && w.pieces > 1) {
          if (in_range) __stcg(p.ws_lse + ws_row(blockIdx.x, w.piece == 0 ? 1 : 0, t, r), -INFINITY);
        }
        if (SPLIT && w.pieces > 1) {
          // Both warpgroups publish their rows, then one thread counts the
          // piece; the CTA that brings the count to `pieces` merges all of
          // them with the log-domain identity lse = ln sum_k e^{lse_k},
          // O = sum_k e^{lse_k - lse} O_k, and resets the counter for the
          // next call.
          // The two rendezvous are bounded mbarrier waits, not bar.sync: if
          // the other warpgroup has aborted, this one gives up too instead
          // of waiting forever.  (The flag is rewritten only after the next
          // item's first rendezvous, which every thread reaches after
          // reading it.)
          __threadfence();
          if (p.stall_site == STALL_SPLIT_SYNC && t == 0) {
            wait_phase(bar(L::NEVER), 0, abort_flag, SITE_INJECTED);
            break;
          }
          if (!softmax_sync()) break;
          if (threadIdx.x == 0) {
            const unsigned int done = atomicAdd(p.ws_count + w.unit, 1u);
            const int last = (done == static_cast<unsigned int>(w.pieces - 1)) ? 1 : 0;
            if (last) p.ws_count[w.unit] = 0u;
            *last_flag = last;
          }
          if (!softmax_sync()) break;
          const bool last = *last_flag != 0;
          const int n_unit = t ? (w.q0 + BLOCK_M < p.Nq) : 1;  // does tile t have rows at all
          if (last && n_unit) {
            // This CTA finished the unit's last piece.  Its own piece is still
            // in TMEM; the others are read from their slots (coalesced: one
            // column of 32 rows per warp load), all loads of a piece issued
            // before any is used.
            __threadfence();
            tc_fence_after();
            float lse_max = lse_self;
            for (int k = 0; k < w.pieces; ++k) {
              if (k == w.piece || !in_range) continue;
              lse_max = fmaxf(lse_max, __ldcg(p.ws_lse + ws_row(w.c_first + k, k == 0 ? 1 : 0, t, r)));
            }
            const float w_self = ex2_approx((lse_self - lse_max) * 1.4426950408889634f);
            float wsum = 0.f;
            uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) +
                                                   (static_cast<size_t>(bh) * p.Nq + row) * D);
            // Pieces are summed in piece order whichever CTA merges, and the
            // own piece's values are formed exactly as they were stored, so
            // the result is bit-for-bit the same on every call.
#pragma unroll 1
            for (int h = 0; h < D / 64; ++h) {
              float acc[64];
#pragma unroll
              for (int c = 0; c < 64; ++c) acc[c] = 0.f;
              float hsum = 0.f;
              for (int k = 0; k < w.pieces; ++k) {
                float wk;
                float v[64];
                if (k == w.piece) {
                  wk = w_self;
#pragma unroll
                  for (int c = 0; c < 64; ++c) v[c] = 0.f;
                  if (n > 0) {  // warp-uniform: the tile's own O is in TMEM
                    uint32_t o[32];
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                      tmem_ld32(tO + 64 * h + c0, o);
                      tmem_wait_ld_regs(o);
#pragma unroll
                      for (int c = 0; c < 32; ++c) v[c0 + c] = __uint_as_float(o[c]) * inv_self;
                    }
                  }
                } else {
                  const int slot = k == 0 ? 1 : 0;
                  wk = 0.f;
#pragma unroll
                  for (int c = 0; c < 64; ++c) v[c] = 0.f;
                  if (in_range) {
                    wk = ex2_approx((__ldcg(p.ws_lse + ws_row(w.c_first + k, slot, t, r)) - lse_max) *
                                    1.4426950408889634f);
                    if (wk != 0.f) {  // a piece that saw no key of this row wrote no O
                      const float* src = p.ws_o + ws_o_base(w.c_first + k, slot, t, D) +
                                         static_cast<size_t>(64 * h) * BLOCK_M + r;
#pragma unroll
                      for (int c = 0; c < 64; ++c) v[c] = __ldcg(src + static_cast<size_t>(c) * BLOCK_M);
                    }
                  }
                }
                hsum += wk;
#pragma unroll
                for (int c = 0; c < 64; ++c) acc[c] = fmaf(wk, v[c], acc[c]);
              }
              wsum = hsum;
              const float inv = 1.f / hsum;
              if (in_range) {
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8)
                  orow[8 * h + c8] =
                      make_uint4(pack2<BF16>(acc[8 * c8] * inv, acc[8 * c8 + 1] * inv),
                                 pack2<BF16>(acc[8 * c8 + 2] * inv, acc[8 * c8 + 3] * inv),
                                 pack2<BF16>(acc[8 * c8 + 4] * inv, acc[8 * c8 + 5] * inv),
                                 pack2<BF16>(acc[8 * c8 + 6] * inv, acc[8 * c8 + 7] * inv));
              }
            }
            if (p.lse != nullptr && in_range)
              p.lse[static_cast<size_t>(bh) * p.Nq + row] =
                  lse_max + lg2_approx(wsum) * 0.69314718055994531f;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

}  // namespace attn_sm100
