// Host side of the attention library: argument validation, launch planning,
// TMA tensor-map encoding, kernel launch and the C ABI declared in attn.h.
//
// Validation never falls back to another path: an unsupported input is an
// error code (the pages warn that some attention kernels silently fall back
// to a slow path for unaligned lengths -- YOLO11 x FlashAttention-2,
// kwkr.cn, sections 4.1 and 4.2; here any length is handled by in-kernel
// masking and anything else is rejected loudly).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_bwd_sm100.cuh"
#include "attn_fwd_sm100.cuh"
#include "proj_gemm_sm100.cuh"

namespace {

using attn_sm100::BLOCK_M;
using attn_sm100::BLOCK_N;
using attn_sm100::FwdParams;
using attn_sm100::NUM_THREADS;
using attn_sm100::SmemLayout;

constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sms = 0;
  // [d = 64, d = 128, d = 128 e4m3][bf16][unit, dual-unit, split kernel]: the
  // shared-memory attribute is set
  std::atomic<bool> smem_attr[3][2][3] = {};
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

int check_args(const void* q, const void* k, const void* v, const void* o, const float* lse,
               int B, int H, int Nq, int Nk, int d, float scale, int dtype) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_NULL;
  if (dtype != ATTN_FP16 && dtype != ATTN_BF16) return ATTN_ERR_DTYPE;
  if (d != 64 && d != 128) return ATTN_ERR_HEAD_DIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_SHAPE;
  const long long bh = static_cast<long long>(B) * H;
  const long long nmax = Nq > Nk ? Nq : Nk;
  // element offsets are 64-bit; tensor-map dims must stay below 2^32; the
  // work-unit count must fit an int
  if (bh >= (1LL << 31) || bh * nmax * d >= (1LL << 62) ||
      bh * ceil_div(ceil_div(Nq, BLOCK_M), 2) >= (1LL << 31))
    return ATTN_ERR_SHAPE;
  auto misaligned = [](const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0;
  };
  if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) ||
      (lse != nullptr && misaligned(lse, 4)))
    return ATTN_ERR_ALIGN;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_SCALE;
  return ATTN_OK;
}

// Split mode pays when unit mode leaves the grid ragged (fewer units than
// SMs, or a last wave under 90 % full) and the serial key-tile steps it saves
// per CTA outweigh its own cost: publishing and merging the pieces of a unit
// (the last piece reads every other piece's O back).  The cost, in key-tile
// steps, was fitted to split and unit timings of small problems on B200:
// about 3.5 + 0.56 per piece at d = 64 and 2.5 + 1.03 per piece at d = 128.
// `unit_steps`: key-tile steps of the largest unit-mode unit (nk; under the
// causal mask a heavy query pair plus its light mirror); `piece_steps`: the
// steps of the largest split-mode unit (one query pair).  Under the causal
// mask the merge cost counts 1.3 times (fitted to seven causal shapes, d = 64
// and 128: split lost where the steps saved only just exceeded the plain
// cost, and won 6 % to 2.7x where they exceeded 1.3 times it).
bool split_pays(long long units, long long unit_steps, long long total_steps,
                long long piece_steps, int num_sms, int d, int causal) {
  if (total_steps < 2) return false;
  const long long grid = units < num_sms ? units : num_sms;
  const long long waves = (units + grid - 1) / grid;
  const double eff = static_cast<double>(units) / static_cast<double>(grid * waves);
  if (eff >= 0.9 && units >= num_sms) return false;
  const long long steps_unit = waves * unit_steps;
  const long long grid_s = total_steps < num_sms ? total_steps : num_sms;
  const long long steps_split = (total_steps + grid_s - 1) / grid_s;
  const long long pieces = (piece_steps * grid_s + total_steps - 1) / total_steps;
  const double cost = (d == 64 ? 3.5 + 0.56 * pieces : 2.5 + 1.03 * pieces) * (causal ? 1.3 : 1.0);
  return static_cast<double>(steps_unit - steps_split) > cost;
}

size_t split_workspace_bytes(int grid, int d, long long units) {
  const size_t rows = static_cast<size_t>(grid) * 2 * 2 * BLOCK_M;
  return rows * d * sizeof(float) + rows * sizeof(float) + static_cast<size_t>(units) * 4 + 16;
}

// Key-tile steps of query pair qp in split mode: query tile i sees min(nk, i + 1)
// key tiles under the top-left causal mask, so the pair needs those of its
// last tile; without the mask, nk.
long long split_pair_steps(int qp, int q_tiles, int kv_tiles, int causal) {
  if (!causal) return kv_tiles;
  const int last_tile = (2 * qp + 1 < q_tiles) ? 2 * qp + 1 : 2 * qp;
  return last_tile + 1 < kv_tiles ? last_tile + 1 : kv_tiles;
}

void fill_plan(int B, int H, int Nq, int Nk, int d, int causal, int num_sms, attn_plan_t* out) {
  const int q_tiles = ceil_div(Nq, BLOCK_M);
  const int q_pairs = ceil_div(q_tiles, 2);
  const int kv_tiles = ceil_div(Nk, BLOCK_N);
  const long long BH = static_cast<long long>(B) * H;
  // Unit mode pairs the lone last query tile of two heads into one dual unit
  // when the tile count is odd (non-causal), so no warpgroup idles.
  const bool dual = !causal && (q_tiles % 2 == 1) && BH >= 2;
  const int units_per_head = causal ? (q_pairs + 1) / 2 : (dual ? q_tiles / 2 : q_pairs);
  const long long dual_units = dual ? (BH + 1) / 2 : 0;
  const long long units = BH * units_per_head + dual_units;
  out->num_q_tiles = q_tiles;
  out->num_q_pairs = q_pairs;
  out->num_kv_tiles = kv_tiles;
  out->num_units = static_cast<int>(units);
  out->units_per_head = units_per_head;
  out->dual_units = static_cast<int>(dual_units);
  out->grid = static_cast<int>(units < num_sms ? units : num_sms);
  out->block = NUM_THREADS;
  out->smem_bytes = d == 64 ? SmemLayout<64>::BYTES : SmemLayout<128>::BYTES;
  out->stages = d == 64 ? SmemLayout<64>::K_STAGES + SmemLayout<64>::V_STAGES
                        : SmemLayout<128>::K_STAGES + SmemLayout<128>::V_STAGES;
  // score tiles per (batch, head): the same count the kernel's work units visit
  long long per_head = 0;
  for (int qt = 0; qt < q_tiles; ++qt) {
    if (causal) {
      const int last_row = (qt * BLOCK_M + BLOCK_M - 1 < Nq - 1) ? qt * BLOCK_M + BLOCK_M - 1 : Nq - 1;
      const int n = last_row / BLOCK_N + 1;
      per_head += n < kv_tiles ? n : kv_tiles;
    } else {
      per_head += kv_tiles;
    }
  }
  out->qk_tile_products = per_head * B * H;
  // split mode keeps plain units (one (batch, head) and query pair each)
  const long long split_units = BH * q_pairs;
  long long steps_per_head = 0, piece_steps = 0, unit_steps = 0;
  for (int qp = 0; qp < q_pairs; ++qp) {
    const long long s = split_pair_steps(qp, q_tiles, kv_tiles, causal);
    steps_per_head += s;
    piece_steps = s > piece_steps ? s : piece_steps;
  }
  if (causal) {  // a unit-mode unit streams a heavy pair and its light mirror
    for (int b = 0; b < units_per_head; ++b) {
      const int heavy = q_pairs - 1 - b;
      const long long s = split_pair_steps(heavy, q_tiles, kv_tiles, 1) +
                          (heavy != b ? split_pair_steps(b, q_tiles, kv_tiles, 1) : 0);
      unit_steps = s > unit_steps ? s : unit_steps;
    }
  } else {
    unit_steps = kv_tiles;
  }
  const long long total_steps = BH * steps_per_head;
  out->split = split_pays(units, unit_steps, total_steps, piece_steps, num_sms, d, causal) ? 1 : 0;
  out->split_grid = static_cast<int>(total_steps < num_sms ? total_steps : num_sms);
  out->split_units = static_cast<int>(split_units);
  out->split_steps = total_steps;
  out->workspace_bytes =
      out->split ? static_cast<long long>(split_workspace_bytes(out->split_grid, d, split_units)) : 0;
}

// Probe the current device once: compute capability 10.0 and SM count.
int current_device(int* dev_out, DeviceInfo** info_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& info = g_dev[dev];
  if (!info.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    info.supported = (major == 10 && minor == 0);
    info.sms = sms;
    info.probed = true;
  }
  if (!info.supported) return ATTN_ERR_ARCH;
  *dev_out = dev;
  *info_out = &info;
  return ATTN_OK;
}

// Internal element-type code of e4m3 operands (attn_fwd_fp8): keeps their
// cached tensor maps apart from 16-bit maps of the same buffers.
constexpr int kDtypeE4M3 = 2;

// 3-D view (cols, rows, B*H) of a [B, H, rows, cols] tensor; boxes of 128
// bytes x 128 rows (64 fp16 / bf16 or 128 e4m3 columns) with the 128-byte
// swizzle the tcgen05 descriptors expect.  Rows past `rows` and columns past
// `cols` read as zero, so ragged tails never touch the next head.
bool encode_rows(CUtensorMap* map, const void* ptr, long long rows, long long BH, int cols,
                 int dtype) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t elem = dtype == kDtypeE4M3 ? 1 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * elem,
                                 static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols) * elem};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(BLOCK_M), 1};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  const CUtensorMapDataType type = dtype == kDtypeE4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = enc(map, type, 3, const_cast<void*>(ptr), dims, strides, box, elem_strides,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B, H, N, d] Q, K or V
bool encode_map(CUtensorMap* map, const void* ptr, int N, long long BH, int d, int dtype) {
  return encode_rows(map, ptr, N, BH, d, dtype);
}

// Per-thread cache of recent calls' tensor maps: repeated calls on the same
// buffers (the common case in a model loop, and every chunk of the pipelined
// host entry) skip the ~µs host encode.  Entries are replaced round robin.
struct MapCache {
  const void* q = nullptr;
  const void* k = nullptr;
  const void* v = nullptr;
  int Nq = 0, Nk = 0, d = 0, dtype = -1, dev = -1;
  long long BH = 0;
  CUtensorMap mq, mk, mv;
};
constexpr int kMapCacheEntries = 16;
struct MapCacheSet {
  MapCache e[kMapCacheEntries];
  int next = 0;
};
thread_local MapCacheSet t_maps;

// The cached maps for these buffers and sizes, encoding them on a miss;
// nullptr if an encode fails.
const MapCache* cached_maps(const void* q, const void* k, const void* v, int Nq, int Nk,
                            long long BH, int d, int dtype, int dev) {
  MapCacheSet& set = t_maps;
  for (const MapCache& mc : set.e)
    if (mc.q == q && mc.k == k && mc.v == v && mc.Nq == Nq && mc.Nk == Nk && mc.d == d &&
        mc.dtype == dtype && mc.dev == dev && mc.BH == BH)
      return &mc;
  MapCache& mc = set.e[set.next];
  set.next = (set.next + 1) % kMapCacheEntries;
  mc.q = nullptr;  // invalid until all three encodes succeed
  // e4m3: v is Vt [B, H, d, Nk], read in tiles of 128 keys x d rows
  if (!encode_map(&mc.mq, q, Nq, BH, d, dtype) || !encode_map(&mc.mk, k, Nk, BH, d, dtype) ||
      !(dtype == kDtypeE4M3 ? encode_rows(&mc.mv, v, d, BH, Nk, dtype)
                            : encode_map(&mc.mv, v, Nk, BH, d, dtype)))
    return nullptr;
  mc.q = q; mc.k = k; mc.v = v;
  mc.Nq = Nq; mc.Nk = Nk; mc.d = d; mc.dtype = dtype; mc.dev = dev; mc.BH = BH;
  return &mc;
}

template <int D, bool BF16, bool SPLIT, bool DUAL, bool FP8>
int launch_one(const MapCache& maps, const FwdParams& prm, int grid, DeviceInfo& info,
               cudaStream_t stream) {
  auto kernel = attn_sm100::attn_fwd_kernel<D, BF16, SPLIT, DUAL, FP8>;
  constexpr int smem = SmemLayout<D, FP8>::BYTES;
  std::atomic<bool>& attr =
      info.smem_attr[FP8 ? 2 : (D == 128 ? 1 : 0)][BF16][SPLIT ? 2 : (DUAL ? 1 : 0)];
  if (!attr.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!attr.load(std::memory_order_relaxed)) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      attr.store(true, std::memory_order_release);
    }
  }
  kernel<<<grid, NUM_THREADS, smem, stream>>>(maps.mq, maps.mk, maps.mv, prm);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Split mode and unit mode with dual units are separate instantiations, so
// the plain unit-mode kernel carries none of their bookkeeping.
template <int D, bool BF16, bool FP8 = false>
int launch(const MapCache& maps, const FwdParams& prm, int grid, DeviceInfo& info,
           cudaStream_t stream) {
  if (prm.split) return launch_one<D, BF16, true, false, FP8>(maps, prm, grid, info, stream);
  if (prm.dual_base >= 0)
    return launch_one<D, BF16, false, true, FP8>(maps, prm, grid, info, stream);
  return launch_one<D, BF16, false, false, FP8>(maps, prm, grid, info, stream);
}

// The extra arguments of the e4m3 forward.
struct Fp8Scales {
  float q_descale, k_descale, v_descale;
};

// `f8` != nullptr: e4m3 operands (q, k and v = Vt), bf16 output; `dtype` is
// then ATTN_BF16, the output type, and the caller has validated the e4m3
// arguments.
static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int Nq, int Nk, int d, float scale, int causal, int dtype,
                    void* workspace, size_t workspace_bytes, attn_stream_t stream,
                    int stall_site = 0, const Fp8Scales* f8 = nullptr) {
  int st = check_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, dtype);
  if (st != ATTN_OK) return st;
  int dev = -1;
  DeviceInfo* info = nullptr;
  st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;

  attn_plan_t plan;
  fill_plan(B, H, Nq, Nk, d, causal, info->sms, &plan);
  const long long BH = static_cast<long long>(B) * H;

  const MapCache* maps = cached_maps(q, k, v, Nq, Nk, BH, d, f8 ? kDtypeE4M3 : dtype, dev);
  if (maps == nullptr) return ATTN_ERR_CUDA;
  const MapCache& mc = *maps;

  FwdParams prm;
  prm.o = o;
  prm.lse = lse;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.BH = static_cast<int>(BH);
  prm.num_q_pairs = plan.num_q_pairs;
  prm.num_kv_tiles = plan.num_kv_tiles;
  prm.units_per_head = plan.units_per_head;
  prm.num_units = plan.num_units;
  prm.dual_base = plan.dual_units > 0 ? plan.num_units - plan.dual_units : -1;
  prm.last_q0 = (plan.num_q_tiles - 1) * BLOCK_M;
  prm.causal = causal ? 1 : 0;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634 *
                                      (f8 ? static_cast<double>(f8->q_descale) * f8->k_descale : 1.0));
  prm.o_scale = f8 ? f8->v_descale : 1.f;
  prm.split = 0;
  prm.total_steps = 0;
  prm.num_q_tiles = plan.num_q_tiles;
  prm.steps_per_head = plan.split_steps / BH;
  prm.ws_o = nullptr;
  prm.ws_lse = nullptr;
  prm.ws_count = nullptr;
  prm.stall_site = stall_site;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int grid = plan.grid;
  if (plan.split && workspace != nullptr &&
      workspace_bytes >= static_cast<size_t>(plan.workspace_bytes) &&
      (reinterpret_cast<uintptr_t>(workspace) & 15) == 0) {
    grid = plan.split_grid;
    const size_t rows = static_cast<size_t>(grid) * 2 * 2 * BLOCK_M;
    char* ws = static_cast<char*>(workspace);
    prm.split = 1;
    // split mode walks plain units: one (batch, head) and query pair each
    prm.units_per_head = plan.num_q_pairs;
    prm.num_units = plan.split_units;
    prm.dual_base = -1;
    prm.total_steps = plan.split_steps;
    prm.ws_o = reinterpret_cast<float*>(ws);
    prm.ws_lse = reinterpret_cast<float*>(ws + rows * d * sizeof(float));
    // the piece counters start at zero (the caller zero-fills a new
    // workspace) and every completed call leaves them at zero again
    prm.ws_count = reinterpret_cast<unsigned int*>(ws + rows * (d + 1) * sizeof(float));
  }
  if (f8) return launch<128, true, true>(mc, prm, grid, *info, s);
  if (d == 64)
    return dtype == ATTN_BF16 ? launch<64, true>(mc, prm, grid, *info, s)
                              : launch<64, false>(mc, prm, grid, *info, s);
  return dtype == ATTN_BF16 ? launch<128, true>(mc, prm, grid, *info, s)
                            : launch<128, false>(mc, prm, grid, *info, s);
}

}  // namespace

// ---------------------------------------------------------------------------
// Pipelined host entry: three non-blocking streams and the events that chain
// them, created once per device on first use (with that device current) and
// kept for the life of the process.  One mutex per device serialises the
// enqueue of concurrent host-entry calls on the shared streams.
constexpr int kHostPipeMaxChunks = 8;
constexpr size_t kHostPipeMinChunkBytes = 2u << 20;  // input bytes below which a chunk is not worth it

struct HostPipe {
  bool ready = false;
  std::mutex mu;
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, end = nullptr, h2d_end = nullptr, comp_end = nullptr;
  cudaEvent_t in_done[kHostPipeMaxChunks] = {}, comp_done[kHostPipeMaxChunks] = {};
};
HostPipe g_host_pipe[kMaxDevices];

int host_pipe(int dev, HostPipe** out) {
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  HostPipe& hp = g_host_pipe[dev];
  if (!hp.ready) {
    const unsigned int ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.end, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.h2d_end, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.comp_end, ef) == cudaSuccess;
    for (int c = 0; ok && c < kHostPipeMaxChunks; ++c)
      ok = cudaEventCreateWithFlags(&hp.in_done[c], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.comp_done[c], ef) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    hp.ready = true;
  }
  *out = &hp;
  return ATTN_OK;
}

// Chunks for a problem of bh (batch, head) slices: up to kHostPipeMaxChunks,
// each with at least kHostPipeMinChunkBytes of input.
int host_pipe_chunks(long long bh, size_t q_head, size_t kv_head) {
  const size_t in_bytes = static_cast<size_t>(bh) * (q_head + 2 * kv_head);
  long long c = static_cast<long long>(in_bytes / kHostPipeMinChunkBytes);
  if (c > kHostPipeMaxChunks) c = kHostPipeMaxChunks;
  if (c > bh) c = bh;
  return c < 1 ? 1 : static_cast<int>(c);
}

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int Nq, int Nk, int d, float scale, int causal, int dtype, attn_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, nullptr, 0, stream);
}

int attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int Nq, int Nk, int d, float scale, int causal, int dtype, void* workspace,
                size_t workspace_bytes, attn_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, workspace,
                  workspace_bytes, stream);
}

int attn_fwd_stall_test(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int Nq, int Nk, int d, float scale, int causal, int dtype,
                        void* workspace, size_t workspace_bytes, int stall_site,
                        attn_stream_t stream) {
  if (stall_site < 1 || stall_site > 4) return ATTN_ERR_SHAPE;
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, workspace,
                  workspace_bytes, stream, stall_site);
}

int attn_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse, int B, int H,
                 int Nq, int Nk, int d, float scale, float q_descale, float k_descale,
                 float v_descale, int causal, void* workspace, size_t workspace_bytes,
                 attn_stream_t stream) {
  if (q == nullptr || k == nullptr || vt == nullptr || o == nullptr) return ATTN_ERR_NULL;
  if (d != 128) return ATTN_ERR_HEAD_DIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || Nk % 16 != 0) return ATTN_ERR_SHAPE;
  for (float f : {q_descale, k_descale, v_descale})
    if (!std::isfinite(f) || !(f > 0.f)) return ATTN_ERR_SCALE;
  // the folded score scale must stay a finite, positive fp32 value
  const double sl2 = static_cast<double>(scale) * q_descale * k_descale;
  if (!std::isfinite(scale) || !(sl2 > 1e-30) || !(sl2 < 1e30)) return ATTN_ERR_SCALE;
  const Fp8Scales f8{q_descale, k_descale, v_descale};
  return fwd_impl(q, k, vt, o, lse, B, H, Nq, Nk, d, scale, causal, ATTN_BF16, workspace,
                  workspace_bytes, stream, 0, &f8);
}

int attn_workspace_size(int B, int H, int Nq, int Nk, int d, int causal, size_t* bytes) {
  if (bytes == nullptr) return ATTN_ERR_NULL;
  if (d != 64 && d != 128) return ATTN_ERR_HEAD_DIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_SHAPE;
  int dev = -1;
  DeviceInfo* info = nullptr;
  const int st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;
  attn_plan_t plan;
  fill_plan(B, H, Nq, Nk, d, causal, info->sms, &plan);
  *bytes = static_cast<size_t>(plan.workspace_bytes);
  return ATTN_OK;
}

int attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                  float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                  float* lse_dev, void* workspace, size_t workspace_bytes, int B, int H, int Nq,
                  int Nk, int d, float scale, int causal, int dtype, attn_stream_t stream) {
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || o_host == nullptr)
    return ATTN_ERR_NULL;
  int st = check_args(q_dev, k_dev, v_dev, o_dev, lse_dev, B, H, Nq, Nk, d, scale, dtype);
  if (st != ATTN_OK) return st;
  int dev = -1;
  DeviceInfo* info = nullptr;
  st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;
  const long long bh = static_cast<long long>(B) * H;
  const size_t q_head = static_cast<size_t>(Nq) * d * 2, kv_head = static_cast<size_t>(Nk) * d * 2;
  const bool with_lse = lse_host != nullptr && lse_dev != nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  attn_plan_t plan;
  fill_plan(B, H, Nq, Nk, d, causal, info->sms, &plan);
  const bool uses_split = plan.split && workspace != nullptr &&
                          workspace_bytes >= static_cast<size_t>(plan.workspace_bytes);
  const int chunks = host_pipe_chunks(bh, q_head, kv_head);
  if (uses_split || chunks < 2) {
    // one shot on the caller's stream: copies in, forward, copies out
    if (cudaMemcpyAsync(q_dev, q_host, bh * q_head, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(k_dev, k_host, bh * kv_head, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(v_dev, v_host, bh * kv_head, cudaMemcpyHostToDevice, s) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    st = fwd_impl(q_dev, k_dev, v_dev, o_dev, lse_dev, B, H, Nq, Nk, d, scale, causal, dtype,
                  workspace, workspace_bytes, stream);
    if (st != ATTN_OK) return st;
    if (cudaMemcpyAsync(o_host, o_dev, bh * q_head, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        (with_lse && cudaMemcpyAsync(lse_host, lse_dev, bh * Nq * sizeof(float),
                                     cudaMemcpyDeviceToHost, s) != cudaSuccess)) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  }

  // Pipelined over chunks of consecutive (batch, head) slices, which are
  // contiguous in every tensor: chunk c's host->device copies, its forward
  // and its device->host copies run on three library streams, so the copies
  // of one chunk overlap the compute and the opposite-direction copies of
  // the others.  Unit mode computes every row the same way whichever unit
  // holds it, so the result is bit-for-bit that of attn_fwd.
  HostPipe* hp = nullptr;
  st = host_pipe(dev, &hp);
  if (st != ATTN_OK) return st;
  std::lock_guard<std::mutex> lock(hp->mu);
  const long long per = (bh + chunks - 1) / chunks;
  // Joins the three library streams back into the caller's stream, so that
  // work the caller enqueues afterwards (or a host wait before it frees or
  // reuses the pinned buffers) follows everything this call enqueued -- on
  // success and on every error path alike.
  auto join = [&]() -> bool {
    return cudaEventRecord(hp->h2d_end, hp->h2d) == cudaSuccess &&
           cudaEventRecord(hp->comp_end, hp->comp) == cudaSuccess &&
           cudaStreamWaitEvent(hp->d2h, hp->h2d_end, 0) == cudaSuccess &&
           cudaStreamWaitEvent(hp->d2h, hp->comp_end, 0) == cudaSuccess &&
           cudaEventRecord(hp->end, hp->d2h) == cudaSuccess &&
           cudaStreamWaitEvent(s, hp->end, 0) == cudaSuccess;
  };
  bool ok = cudaEventRecord(hp->start, s) == cudaSuccess &&
            cudaStreamWaitEvent(hp->h2d, hp->start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hp->comp, hp->start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hp->d2h, hp->start, 0) == cudaSuccess;
  if (!ok) {  // nothing of this call is enqueued yet
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  for (int c = 0; ok && st == ATTN_OK && c < chunks; ++c) {
    const long long h0 = c * per;
    const long long nh = (h0 + per <= bh) ? per : bh - h0;
    if (nh <= 0) break;
    const size_t qo = static_cast<size_t>(h0) * q_head, kvo = static_cast<size_t>(h0) * kv_head;
    const size_t lo = static_cast<size_t>(h0) * Nq;
    ok = cudaMemcpyAsync(static_cast<char*>(q_dev) + qo, static_cast<const char*>(q_host) + qo,
                         nh * q_head, cudaMemcpyHostToDevice, hp->h2d) == cudaSuccess &&
         cudaMemcpyAsync(static_cast<char*>(k_dev) + kvo, static_cast<const char*>(k_host) + kvo,
                         nh * kv_head, cudaMemcpyHostToDevice, hp->h2d) == cudaSuccess &&
         cudaMemcpyAsync(static_cast<char*>(v_dev) + kvo, static_cast<const char*>(v_host) + kvo,
                         nh * kv_head, cudaMemcpyHostToDevice, hp->h2d) == cudaSuccess &&
         cudaEventRecord(hp->in_done[c], hp->h2d) == cudaSuccess &&
         cudaStreamWaitEvent(hp->comp, hp->in_done[c], 0) == cudaSuccess;
    if (!ok) break;
    st = fwd_impl(static_cast<char*>(q_dev) + qo, static_cast<char*>(k_dev) + kvo,
                  static_cast<char*>(v_dev) + kvo, static_cast<char*>(o_dev) + qo,
                  lse_dev != nullptr ? lse_dev + lo : nullptr, static_cast<int>(nh), 1, Nq, Nk, d,
                  scale, causal, dtype, nullptr, 0, reinterpret_cast<attn_stream_t>(hp->comp));
    if (st != ATTN_OK) break;
    ok = cudaEventRecord(hp->comp_done[c], hp->comp) == cudaSuccess &&
         cudaStreamWaitEvent(hp->d2h, hp->comp_done[c], 0) == cudaSuccess &&
         cudaMemcpyAsync(static_cast<char*>(o_host) + qo, static_cast<char*>(o_dev) + qo,
                         nh * q_head, cudaMemcpyDeviceToHost, hp->d2h) == cudaSuccess &&
         (!with_lse || cudaMemcpyAsync(lse_host + lo, lse_dev + lo, nh * Nq * sizeof(float),
                                       cudaMemcpyDeviceToHost, hp->d2h) == cudaSuccess);
  }
  if (!ok) {
    cudaGetLastError();
    st = ATTN_ERR_CUDA;
  }
  if (!join()) {
    cudaGetLastError();
    if (st == ATTN_OK) st = ATTN_ERR_CUDA;
  }
  return st;
}

int attn_plan(int B, int H, int Nq, int Nk, int d, int causal, int num_sms, attn_plan_t* out) {
  if (out == nullptr) return ATTN_ERR_NULL;
  if (d != 64 && d != 128) return ATTN_ERR_HEAD_DIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || num_sms < 1) return ATTN_ERR_SHAPE;
  const long long bh = static_cast<long long>(B) * H;
  if (bh >= (1LL << 31) || bh * ceil_div(ceil_div(Nq, BLOCK_M), 2) >= (1LL << 31))
    return ATTN_ERR_SHAPE;
  fill_plan(B, H, Nq, Nk, d, causal, num_sms, out);
  return ATTN_OK;
}

int attn_get_device_status(attn_stream_t stream, unsigned int* detail) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, attn_sm100::g_attn_status, sizeof(word)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  if (detail != nullptr) *detail = word;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(attn_sm100::g_attn_status, &zero, sizeof(zero)) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_ERR_DEVICE_TIMEOUT;
  }
  return ATTN_OK;
}

const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "success";
    case ATTN_ERR_NULL: return "a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "B, H, Nq and Nk must be >= 1 and the sizes must fit the index range";
    case ATTN_ERR_HEAD_DIM: return "head dimension d must be 64 or 128";
    case ATTN_ERR_DTYPE: return "dtype must be ATTN_FP16 or ATTN_BF16";
    case ATTN_ERR_ALIGN: return "q, k, v, o must be 16-byte aligned and lse 4-byte aligned";
    case ATTN_ERR_SCALE: return "scale must be finite and > 0";
    case ATTN_ERR_ARCH: return "the current device is not compute capability 10.0 (sm_100a)";
    case ATTN_ERR_CUDA: return "a CUDA call failed (no usable device, encode or launch error)";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded internal wait; its output is invalid";
    case ATTN_ERR_SCRATCH_LIMIT: return "the problem needs more scratch than attn_fwd_noalloc's fixed 24 MiB";
    case ATTN_ERR_WORKSPACE: return "the workspace is NULL, smaller than attn_bwd_workspace_size or not 16-byte aligned";
    default: return "unknown status";
  }
}

int attn_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward: row pass, main pass, dQ conversion.
// ---------------------------------------------------------------------------
namespace {

// fp32 dQ accumulator [BH][Nq][d], then lse in base 2 and D, each [BH][Nq_pad].
size_t bwd_workspace_bytes(long long BH, int Nq, int d) {
  const size_t nq_pad = static_cast<size_t>(ceil_div(Nq, BLOCK_M)) * BLOCK_M;
  return static_cast<size_t>(BH) * Nq * d * 4 + 2 * static_cast<size_t>(BH) * nq_pad * 4;
}

struct BwdMapCache {
  const void* dout = nullptr;
  int Nq = 0, d = 0, dtype = -1, dev = -1;
  long long BH = 0;
  CUtensorMap m;
};
thread_local BwdMapCache t_do_map;

std::atomic<bool> g_bwd_attr[kMaxDevices][2][2];  // [dev][d == 128][bf16]

template <int D, bool BF16>
int bwd_launch(const MapCache& maps, const CUtensorMap& m_do, const CUtensorMap& m_dq,
               const void* o, const void* dout,
               const float* lse, void* dq, const attn_sm100::BwdParams& prm, int dev, int sms,
               cudaStream_t stream) {
  using L = attn_sm100::BwdSmem<D>;
  auto main_kernel = attn_sm100::bwd_main_kernel<D, BF16>;
  std::atomic<bool>& attr = g_bwd_attr[dev][D == 128][BF16];
  if (!attr.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!attr.load(std::memory_order_relaxed)) {
      if (cudaFuncSetAttribute(main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::BYTES) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      attr.store(true, std::memory_order_release);
    }
  }
  const long long BH = prm.BH;
  const long long prep_rows = BH * prm.nq_pad;
  const long long prep_blocks_needed = (prep_rows + 31) / 32;  // 32 rows per 256-thread block
  const int prep_blocks = static_cast<int>(prep_blocks_needed < 16LL * sms ? prep_blocks_needed : 16LL * sms);
  attn_sm100::bwd_prep_kernel<D, BF16><<<prep_blocks, 256, 0, stream>>>(
      static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse,
      const_cast<float*>(prm.lse2), const_cast<float*>(prm.dsum), prm.dq_acc, prm.Nq, prm.nq_pad, BH);
  const long long grid = static_cast<long long>(prm.nk_tiles) * BH;
  main_kernel<<<static_cast<unsigned int>(grid), attn_sm100::BWD_THREADS, L::BYTES, stream>>>(
      maps.mq, maps.mk, maps.mv, m_do, m_dq, prm);
  const long long n4 = BH * prm.Nq * (D / 4);
  const long long dq_blocks_needed = (n4 + 255) / 256;
  const int dq_blocks = static_cast<int>(dq_blocks_needed < 16LL * sms ? dq_blocks_needed : 16LL * sms);
  attn_sm100::bwd_dq_kernel<BF16><<<dq_blocks, 256, 0, stream>>>(prm.dq_acc,
                                                                 static_cast<uint16_t*>(dq), n4,
                                                                 prm.scale);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" int attn_bwd_workspace_size(int B, int H, int Nq, int Nk, int d, size_t* bytes) {
  if (bytes == nullptr) return ATTN_ERR_NULL;
  if (d != 64 && d != 128) return ATTN_ERR_HEAD_DIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_SHAPE;
  *bytes = bwd_workspace_bytes(static_cast<long long>(B) * H, Nq, d);
  return ATTN_OK;
}

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                        int H, int Nq, int Nk, int d, float scale, int causal, int dtype,
                        void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  int st = check_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, dtype);
  if (st != ATTN_OK) return st;
  if (lse == nullptr || dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr)
    return ATTN_ERR_NULL;
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) != 0; };
  if (misaligned(dout) || misaligned(dq) || misaligned(dk) || misaligned(dv)) return ATTN_ERR_ALIGN;
  const long long BH = static_cast<long long>(B) * H;
  const int nk_tiles = ceil_div(Nk, BLOCK_N);
  if (BH * nk_tiles >= (1LL << 31)) return ATTN_ERR_SHAPE;
  if (workspace == nullptr || misaligned(workspace) ||
      workspace_bytes < bwd_workspace_bytes(BH, Nq, d))
    return ATTN_ERR_WORKSPACE;
  int dev = -1;
  DeviceInfo* info = nullptr;
  st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;
  const MapCache* maps = cached_maps(q, k, v, Nq, Nk, BH, d, dtype, dev);
  if (maps == nullptr) return ATTN_ERR_CUDA;
  BwdMapCache& dm = t_do_map;
  if (dm.dout != dout || dm.Nq != Nq || dm.d != d || dm.dtype != dtype || dm.dev != dev ||
      dm.BH != BH) {
    dm.dout = nullptr;
    if (!encode_map(&dm.m, dout, Nq, BH, d, dtype)) return ATTN_ERR_CUDA;
    dm.dout = dout; dm.Nq = Nq; dm.d = d; dm.dtype = dtype; dm.dev = dev; dm.BH = BH;
  }
  attn_sm100::BwdParams prm;
  const int nq_tiles = ceil_div(Nq, BLOCK_M);
  const int nq_pad = nq_tiles * BLOCK_M;
  char* ws = static_cast<char*>(workspace);
  prm.dk = dk;
  prm.dv = dv;
  prm.dq_acc = reinterpret_cast<float*>(ws);
  prm.lse2 = reinterpret_cast<const float*>(ws + static_cast<size_t>(BH) * Nq * d * 4);
  prm.dsum = prm.lse2 + static_cast<size_t>(BH) * nq_pad;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.BH = static_cast<int>(BH);
  prm.nq_tiles = nq_tiles;
  prm.nk_tiles = nk_tiles;
  prm.nq_pad = nq_pad;
  prm.causal = causal ? 1 : 0;
  prm.scale = scale;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the fp32 dQ accumulator as the 3-D map (d, Nq, B H) with 32-column x
  // 128-row boxes and the 128-byte swizzle, the target of the bulk reductions
  CUtensorMap m_dq;
  {
    EncodeTiledFn enc = encode_fn();
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Nq),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                   static_cast<cuuint64_t>(Nq) * d * 4};
    const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(BLOCK_M), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc == nullptr ||
        enc(&m_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, prm.dq_acc, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ATTN_ERR_CUDA;
  }
  if (d == 64)
    return dtype == ATTN_BF16
               ? bwd_launch<64, true>(*maps, dm.m, m_dq, o, dout, lse, dq, prm, dev, info->sms, s)
               : bwd_launch<64, false>(*maps, dm.m, m_dq, o, dout, lse, dq, prm, dev, info->sms, s);
  return dtype == ATTN_BF16
             ? bwd_launch<128, true>(*maps, dm.m, m_dq, o, dout, lse, dq, prm, dev, info->sms, s)
             : bwd_launch<128, false>(*maps, dm.m, m_dq, o, dout, lse, dq, prm, dev, info->sms, s);
}

// ---------------------------------------------------------------------------
// Projections of the attention block (QKV in, output out), fused with the
// [B, H, N, d] layout of the attention.
// ---------------------------------------------------------------------------
namespace {

// Tiled map of a 16-bit tensor of `rank` dims (innermost first), strides in
// bytes for dims 1.., boxes of 64 x 128 (x 1 ...) with the 128-byte swizzle.
bool encode_tiled(CUtensorMap* map, const void* ptr, int rank, const cuuint64_t* dims,
                  const cuuint64_t* strides, int dtype) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint32_t box[5] = {64, 128, 1, 1, 1};
  const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  return enc(map, dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
             rank, const_cast<void*>(ptr), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, cols] row-major 16-bit matrix as the 3-D map (cols, rows, 1).
bool encode_matrix(CUtensorMap* map, const void* ptr, long long rows, long long cols, int dtype) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 1};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2,
                                 static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols) * 2};
  return encode_tiled(map, ptr, 3, dims, strides, dtype);
}

std::atomic<bool> g_proj_attr[kMaxDevices][2][2];  // [dev][bf16][mode]

template <bool BF16, int MODE>
int proj_launch(const CUtensorMap& ma, const CUtensorMap& mb, const attn_sm100::ProjParams& prm,
                int m_tiles_total, int dev, cudaStream_t stream) {
  auto kernel = attn_sm100::proj_gemm_kernel<BF16, MODE>;
  constexpr int smem = attn_sm100::ProjSmem::BYTES;
  std::atomic<bool>& attr = g_proj_attr[dev][BF16][MODE];
  if (!attr.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!attr.load(std::memory_order_relaxed)) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_CUDA;
      }
      attr.store(true, std::memory_order_release);
    }
  }
  const dim3 grid(static_cast<unsigned int>(ceil_div(prm.N_out, 128)),
                  static_cast<unsigned int>(m_tiles_total));
  kernel<<<grid, attn_sm100::PROJ_THREADS, smem, stream>>>(ma, mb, prm);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

int check_proj_shape(int B, int N, int H, int d, int dtype) {
  if (dtype != ATTN_FP16 && dtype != ATTN_BF16) return ATTN_ERR_DTYPE;
  if (d != 64 && d != 128) return ATTN_ERR_HEAD_DIM;
  if (B < 1 || N < 1 || H < 1) return ATTN_ERR_SHAPE;
  const long long rows = static_cast<long long>(B) * N;
  if (rows >= (1LL << 31) / 2 || static_cast<long long>(H) * d * 3 >= (1LL << 30) ||
      (rows + 127) / 128 >= 65535)
    return ATTN_ERR_SHAPE;
  return ATTN_OK;
}

int qkv_proj_impl(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k, void* v,
                  int B, int N, int H, int d, int dtype, cudaStream_t s) {
  int st = check_proj_shape(B, N, H, d, dtype);
  if (st != ATTN_OK) return st;
  if (x == nullptr || w_qkv == nullptr || q == nullptr || k == nullptr || v == nullptr)
    return ATTN_ERR_NULL;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (b_qkv != nullptr && (reinterpret_cast<uintptr_t>(b_qkv) & 3) != 0))
    return ATTN_ERR_ALIGN;
  int dev = -1;
  DeviceInfo* info = nullptr;
  st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;
  const int C = H * d;
  const long long M = static_cast<long long>(B) * N;
  CUtensorMap ma, mb;
  if (!encode_matrix(&ma, x, M, C, dtype) || !encode_matrix(&mb, w_qkv, 3LL * C, C, dtype))
    return ATTN_ERR_CUDA;
  attn_sm100::ProjParams prm;
  prm.bias = b_qkv;
  prm.out0 = q;
  prm.out1 = k;
  prm.out2 = v;
  prm.B = B;
  prm.N = N;
  prm.K = C;
  prm.N_out = 3 * C;
  prm.H = H;
  prm.d = d;
  prm.m_tiles = static_cast<int>((M + 127) / 128);
  return dtype == ATTN_BF16
             ? proj_launch<true, attn_sm100::PROJ_QKV>(ma, mb, prm, prm.m_tiles, dev, s)
             : proj_launch<false, attn_sm100::PROJ_QKV>(ma, mb, prm, prm.m_tiles, dev, s);
}

int out_proj_impl(const void* o, const void* w_o, const float* b_o, void* y, int B, int N, int H,
                  int d, int C_out, int dtype, cudaStream_t s) {
  int st = check_proj_shape(B, N, H, d, dtype);
  if (st != ATTN_OK) return st;
  if (C_out < 8 || C_out % 8 != 0 || C_out >= (1 << 30)) return ATTN_ERR_SHAPE;
  if (static_cast<long long>(B) * ceil_div(N, 128) >= 65535) return ATTN_ERR_SHAPE;  // grid rows
  if (o == nullptr || w_o == nullptr || y == nullptr) return ATTN_ERR_NULL;
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(y) ||
      (b_o != nullptr && (reinterpret_cast<uintptr_t>(b_o) & 3) != 0))
    return ATTN_ERR_ALIGN;
  int dev = -1;
  DeviceInfo* info = nullptr;
  st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;
  const int C = H * d;
  CUtensorMap ma, mb;
  // o [B, H, N, d] as the 4-D map (d, N, H, B): box (64, 128, 1, 1) is 128 rows of
  // o' = [B N, H d] over 64 of its columns, inside one head
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2,
                                 static_cast<cuuint64_t>(H) * N * d * 2};
  if (!encode_tiled(&ma, o, 4, dims, strides, dtype) || !encode_matrix(&mb, w_o, C_out, C, dtype))
    return ATTN_ERR_CUDA;
  attn_sm100::ProjParams prm;
  prm.bias = b_o;
  prm.out0 = y;
  prm.out1 = prm.out2 = nullptr;
  prm.B = B;
  prm.N = N;
  prm.K = C;
  prm.N_out = C_out;
  prm.H = H;
  prm.d = d;
  prm.m_tiles = ceil_div(N, 128);
  const int m_total = B * prm.m_tiles;
  return dtype == ATTN_BF16 ? proj_launch<true, attn_sm100::PROJ_OUT>(ma, mb, prm, m_total, dev, s)
                            : proj_launch<false, attn_sm100::PROJ_OUT>(ma, mb, prm, m_total, dev, s);
}

}  // namespace

extern "C" int attn_qkv_proj(const void* x, const void* w_qkv, const float* b_qkv, void* q,
                             void* k, void* v, int B, int N, int H, int d, int dtype,
                             attn_stream_t stream) {
  return qkv_proj_impl(x, w_qkv, b_qkv, q, k, v, B, N, H, d, dtype,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int attn_out_proj(const void* o, const void* w_o, const float* b_o, void* y, int B,
                             int N, int H, int d, int C_out, int dtype, attn_stream_t stream) {
  return out_proj_impl(o, w_o, b_o, y, B, N, H, d, C_out, dtype,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int attn_block_fwd(const void* x, const void* w_qkv, const float* b_qkv,
                              const void* w_o, const float* b_o, void* q, void* k, void* v,
                              void* o, float* lse, void* y, int B, int N, int H, int d,
                              int C_out, float scale, int causal, int dtype,
                              attn_stream_t stream) {
  // every argument is checked before the first launch
  int st = check_proj_shape(B, N, H, d, dtype);
  if (st != ATTN_OK) return st;
  if (C_out < 8 || C_out % 8 != 0) return ATTN_ERR_SHAPE;
  if (x == nullptr || w_qkv == nullptr || w_o == nullptr || y == nullptr) return ATTN_ERR_NULL;
  st = check_args(q, k, v, o, lse, B, H, N, N, d, scale, dtype);
  if (st != ATTN_OK) return st;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(w_o) || !aligned16(y) ||
      (b_qkv != nullptr && (reinterpret_cast<uintptr_t>(b_qkv) & 3) != 0) ||
      (b_o != nullptr && (reinterpret_cast<uintptr_t>(b_o) & 3) != 0))
    return ATTN_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = qkv_proj_impl(x, w_qkv, b_qkv, q, k, v, B, N, H, d, dtype, s);
  if (st != ATTN_OK) return st;
  st = fwd_impl(q, k, v, o, lse, B, H, N, N, d, scale, causal, dtype, nullptr, 0, stream);
  if (st != ATTN_OK) return st;
  return out_proj_impl(o, w_o, b_o, y, B, N, H, d, C_out, dtype, s);
}

// ---------------------------------------------------------------------------
// Allocation-free entry point.
//
// Some callers cannot allocate device memory at all: a plugin running inside
// a framework that owns every byte of device memory through its own
// allocator, a deployment whose memory plan is fixed before it starts, or a
// latency-critical path where cudaMalloc's implicit device synchronisation
// would stall other streams.  For them attn_fwd_noalloc takes its split-mode
// workspace from the fixed array below instead of from the caller.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 24u << 20;  // 24 MiB

// Split-mode workspace of attn_fwd_noalloc.  Every GPU that loads this library
// holds these 24 MiB until the process exits.  In host code the name is only
// a stand-in: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_ptr[kMaxDevices] = {};  // device address per device, guarded by g_dev_mutex

// First call on a device: look up the array's device address with that device
// current (this is why the first call should come before any stream capture).
int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int Nq, int Nk, int d, float scale, int causal,
                                int dtype, attn_stream_t stream) {
  int st = check_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, dtype);
  if (st != ATTN_OK) return st;
  int dev = -1;
  DeviceInfo* info = nullptr;
  st = current_device(&dev, &info);
  if (st != ATTN_OK) return st;
  attn_plan_t plan;
  fill_plan(B, H, Nq, Nk, d, causal, info->sms, &plan);
  if (!plan.split)  // this shape needs no scratch at all
    return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, nullptr, 0, stream);
  if (static_cast<size_t>(plan.workspace_bytes) > kNoAllocScratchBytes) return ATTN_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  st = noalloc_scratch(dev, &ws);
  if (st != ATTN_OK) return st;
  // The array keeps the previous call's contents; the piece counters must
  // start at zero (a call that timed out may have left them set).
  const size_t rows = static_cast<size_t>(plan.split_grid) * 2 * 2 * BLOCK_M;
  char* counters = static_cast<char*>(ws) + rows * (d + 1) * sizeof(float);
  if (cudaMemsetAsync(counters, 0, static_cast<size_t>(plan.split_units) * 4,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, ws,
                  kNoAllocScratchBytes, stream);
}
