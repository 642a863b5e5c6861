/*
 * attn.h -- C ABI of the B200 (sm_100a) exact attention forward.
 *
 *   O = softmax(Q K^T * scale [+ causal mask]) V,    lse = logsumexp of the scaled scores
 *
 * The operation is the attention formula of "FlashAttention 深度解读：让大模型注意力机制
 * 一口气算完" (coreui.cn), section "背景", computed by the tiled online softmax of its section
 * "原理" and of the YOLO11 x FlashAttention-2 page (kwkr.cn), section 1.2: the N x N score
 * matrix never reaches HBM.  The argument list mirrors the pages' Python entry points,
 * torch's scaled_dot_product_attention(q, k, v, is_causal, scale) (kwkr.cn, section 2.2) and
 * flash_attention(q, k, v, causal) (coreui.cn, section "怎么用"); dropout is not supported
 * (inference, dropout_p = 0).
 *
 * Conventions shared by every entry point:
 *   - Tensors are contiguous row-major.  q is [B, H, Nq, d]; k and v are [B, H, Nk, d];
 *     o is [B, H, Nq, d], all in `dtype` (ATTN_FP16 or ATTN_BF16).  lse is [B, H, Nq]
 *     float32, natural log: lse[i] = ln(sum_j exp(scale * q_i . k_j)) over the visible keys.
 *   - causal != 0 applies the top-left aligned mask: query i sees key j iff j <= i (the
 *     convention of torch's is_causal).  Every query row sees at least key 0.
 *   - scale is the factor applied to Q K^T; the usual value is 1/sqrt(d).
 *   - All memory is owned by the caller.  The library allocates nothing per call.  The one
 *     exception is attn_fwd_noalloc, which uses a fixed scratch array inside the library
 *     (see its declaration).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default stream).  A
 *     return of ATTN_OK means the arguments were valid and the kernel was enqueued.
 *   - No fallback path exists: an unsupported input returns an error code; nothing is
 *     computed a different way.
 *   - Thread safety: calls from several host threads are safe, except that calls of
 *     attn_fwd_noalloc that overlap on the GPU race on its shared scratch array (see its
 *     declaration).
 */
#ifndef ATTN_SM100_ATTN_H_
#define ATTN_SM100_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
  ATTN_FP16 = 0,
  ATTN_BF16 = 1
} attn_dtype_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_NULL = 1,           /* a required pointer is NULL */
  ATTN_ERR_SHAPE = 2,          /* B, H, Nq or Nk < 1, or the sizes overflow the index range */
  ATTN_ERR_HEAD_DIM = 3,       /* d is not 64 or 128 */
  ATTN_ERR_DTYPE = 4,          /* dtype is not ATTN_FP16 / ATTN_BF16 */
  ATTN_ERR_ALIGN = 5,          /* q, k, v, o not 16-byte aligned, or lse not 4-byte aligned */
  ATTN_ERR_SCALE = 6,          /* scale is not finite and > 0 */
  ATTN_ERR_ARCH = 7,           /* current device is not compute capability 10.0 (B200) */
  ATTN_ERR_CUDA = 8,           /* a CUDA runtime / driver call failed (no device, launch error) */
  ATTN_ERR_DEVICE_TIMEOUT = 9, /* a kernel gave up waiting (see attn_get_device_status) */
  ATTN_ERR_SCRATCH_LIMIT = 10,  /* attn_fwd_noalloc: the problem needs more than its fixed scratch */
  ATTN_ERR_WORKSPACE = 11       /* attn_bwd: workspace NULL, smaller than required or not 16-byte aligned */
} attn_status_t;

/* Launch geometry for one call (see attn_plan). */
typedef struct {
  int num_q_tiles;   /* ceil(Nq / 128): 128-row query tiles per (batch, head)            */
  int num_q_pairs;   /* ceil(num_q_tiles / 2): query tiles are processed in pairs         */
  int num_kv_tiles;  /* ceil(Nk / 128): 128-key tiles per (batch, head)                   */
  int units_per_head; /* work units per (batch, head): num_q_pairs; for causal
                         ceil(num_q_pairs / 2) (a heavy query pair with its mirror); with
                         dual units num_q_tiles / 2 (the full query pairs)                  */
  int num_units;     /* B * H * units_per_head + dual_units work units (unit mode)        */
  int dual_units;    /* non-causal, odd num_q_tiles, B * H >= 2: ceil(B * H / 2) units that
                        each pair the lone last query tile of two heads; else 0            */
  int grid;          /* persistent CTAs launched: min(num_units, SM count)                */
  int block;         /* threads per CTA                                                   */
  int smem_bytes;    /* dynamic shared memory per CTA (16-bit operands; attn_fwd_fp8's
                        e4m3 tiles take 4 + 4 ring slots and about 193 KB)                 */
  int stages;        /* K/V shared-memory ring slots (16-bit operands)                    */
  long long qk_tile_products; /* 128x128 score tiles computed (incl. masked tail tiles)   */
  int split;         /* 1 if attn_fwd_ws would use split mode for these sizes (see below)  */
  int split_grid;    /* CTAs launched in split mode: min(SM count, split_steps)             */
  int split_units;   /* units split mode shares out: B * H * num_q_pairs (no dual units)  */
  long long workspace_bytes; /* workspace attn_fwd_ws needs for split mode; 0 if unused    */
  long long split_steps;     /* key-tile steps split mode shares out: sum over the split units
                                of the key tiles each query pair sees                       */
} attn_plan_t;

/*
 * CUDA graphs.  attn_fwd, attn_fwd_ws, attn_fwd_fp8, attn_bwd, attn_qkv_proj, attn_out_proj and
 * attn_block_fwd allocate nothing and never synchronise, so after one ordinary call with the
 * same dtype and head size (which sets the kernel's shared-memory attribute) they can be
 * captured into a CUDA graph on the caller's stream and replayed; split mode resets its piece
 * counters at the end of every call, so a captured workspace stays valid across replays.
 */

/*
 * attn_fwd -- the attention forward on device memory.
 *
 *   q, k, v  device pointers, 16-byte aligned, layouts above, read only.
 *   o        device pointer, 16-byte aligned, [B, H, Nq, d], written (rows < Nq only).
 *   lse      device pointer to [B, H, Nq] float32, 4-byte aligned, written; or NULL to skip.
 *   B, H     batch and heads, >= 1.    Nq, Nk  query and key counts, >= 1 (any value; no
 *            multiple-of-8 or multiple-of-128 requirement -- ragged tails are masked in the
 *            kernel).
 *   d        head dimension, 64 or 128.
 *   scale    softmax scale, finite and > 0.
 *   causal   0 = full attention, nonzero = top-left causal mask.
 *   dtype    ATTN_FP16 or ATTN_BF16 (q, k, v and o share it).
 *   stream   CUDA stream to enqueue on.
 *
 * Returns ATTN_OK after enqueueing.  Argument errors are detected on the host before any
 * CUDA call, in this order: ATTN_ERR_NULL, ATTN_ERR_DTYPE, ATTN_ERR_HEAD_DIM, ATTN_ERR_SHAPE,
 * ATTN_ERR_ALIGN, ATTN_ERR_SCALE; then ATTN_ERR_CUDA (no usable device) or ATTN_ERR_ARCH.
 * On any error nothing is enqueued and o / lse are untouched.  Precision: fp32 accumulation
 * and softmax statistics; P is rounded to `dtype` before the P V product; O is rounded to
 * nearest-even once.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int Nq, int Nk, int d, float scale, int causal, int dtype, attn_stream_t stream);

/*
 * attn_fwd_ws -- attn_fwd with a caller-provided device workspace that enables split mode.
 *
 * For problems whose work units would fill the GPU unevenly (a ragged last wave, or fewer
 * units than SMs) and where the serial key-tile steps this saves outweigh the cost of merging
 * pieces (few units with many key tiles each, e.g. B = H = 1, N = 2000, causal or not;
 * attn_plan reports the decision), the kernel divides the flattened (unit, key tile) range
 * evenly over the CTAs.  A unit is one query pair of one (batch, head) with the key tiles
 * its queries see (under the causal mask a pair's later tile sees i + 1 key tiles for
 * query tile i, its first tile one fewer).  A unit cut by a range boundary
 * is computed in pieces; each piece writes its normalised O and its logsumexp to the
 * workspace and the last piece to finish merges them exactly with the log-domain identity
 * lse = ln sum_k exp(lse_k), O = sum_k exp(lse_k - lse) O_k (the saved-statistics
 * combination of the "log 域" accumulation, coreui.cn section "原理").  Results equal those
 * of attn_fwd up to rounding.
 *
 *   workspace        device pointer, 16-byte aligned, at least attn_workspace_size() bytes,
 *                    caller-owned.  Zero-fill it once before its first use (cudaMemset): it
 *                    holds per-unit piece counters, and every completed call leaves them at
 *                    zero again, so later calls need no clearing.  After a call that ends in
 *                    ATTN_ERR_DEVICE_TIMEOUT the counters may be left non-zero: zero-fill
 *                    the workspace again.  Calls that share a workspace must be ordered
 *                    (same stream); calls that overlap on the GPU with one workspace race.
 *   workspace_bytes  its size.  If the workspace is NULL, too small or misaligned, or split
 *                    mode does not pay for these sizes, the call behaves exactly as attn_fwd.
 * Other arguments, errors and asynchrony as attn_fwd.
 */
int attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int Nq, int Nk, int d, float scale, int causal, int dtype, void* workspace,
                size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_workspace_size -- bytes of workspace attn_fwd_ws uses for these sizes on the current
 * device (0 when split mode is not used).  Errors: ATTN_ERR_NULL (bytes NULL),
 * ATTN_ERR_HEAD_DIM, ATTN_ERR_SHAPE, ATTN_ERR_CUDA / ATTN_ERR_ARCH (no usable device).
 */
int attn_workspace_size(int B, int H, int Nq, int Nk, int d, int causal, size_t* bytes);

/*
 * attn_fwd_fp8 -- attn_fwd_ws with 8-bit floating-point (e4m3) Q, K and V.
 *
 * "一个反直觉的事实：大模型推理的瓶颈不是计算，而是显存" (ai2ai.xin), section
 * "FlashAttention-3的进一步增强", item 2: the attention runs on FP8 operands at half the
 * memory of 16-bit ones.  Each input is an e4m3 tensor with one descale factor: the value
 * an element stands for is e4m3(code) * descale.  The result is the exact attention of those
 * values, O = softmax(scale * Q K^T) V with lse as in attn_fwd, computed with fp32
 * accumulation and softmax statistics; P is rounded to e4m3 (relative error at most 2^-4,
 * absolute at most 2^-10 relative to the running row maximum) before the P V product, and
 * O is rounded once to bf16.
 *
 *   q   device, [B, H, Nq, d] e4m3 codes (one byte each), contiguous.
 *   k   device, [B, H, Nk, d] e4m3 codes, contiguous.
 *   vt  device, V TRANSPOSED: [B, H, d, Nk] e4m3 codes, contiguous (keys innermost, so
 *       both products read their operands along the contracted axis).
 *   o   device, [B, H, Nq, d] bf16 output.  lse as attn_fwd (nullable).
 *   d   128 (the only head size of this entry point).  Nk a multiple of 16 (the byte
 *       stride of a vt row must be a multiple of 16).
 *   q_descale, k_descale, v_descale  finite and > 0; scale * q_descale * k_descale must be
 *       a normal fp32 value.
 *   workspace, workspace_bytes  as attn_fwd_ws (attn_workspace_size with d = 128).
 * Errors, in this order: ATTN_ERR_NULL, ATTN_ERR_HEAD_DIM (d != 128), ATTN_ERR_SHAPE (also
 * Nk % 16 != 0), ATTN_ERR_SCALE (descales), then the checks of attn_fwd (ATTN_ERR_ALIGN:
 * q, k, vt, o 16-byte aligned).  On any error nothing is enqueued.  Asynchrony as attn_fwd.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse, int B, int H,
                 int Nq, int Nk, int d, float scale, float q_descale, float k_descale,
                 float v_descale, int causal, void* workspace, size_t workspace_bytes,
                 attn_stream_t stream);

/*
 * attn_fwd_noalloc -- attn_fwd_ws without a caller workspace and without any allocation.
 *
 * The pages have no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory: a plugin inside a framework that owns all device memory through
 * its own allocator, a deployment whose memory plan is fixed before it runs, or a path where
 * cudaMalloc's implicit device-wide synchronisation would stall other work.  It computes
 * exactly what attn_fwd_ws computes (same kernel, split mode where that pays) but takes the
 * workspace from a fixed 24 MiB array inside the library.  Every GPU that loads the library
 * holds that array until the process exits.
 *
 *   - Arguments, layouts and the other error codes as attn_fwd.  Nothing is allocated: no
 *     cudaMalloc, no cudaFree, no allocating library call.
 *   - Returns ATTN_ERR_SCRATCH_LIMIT, without enqueueing anything, when split mode would need
 *     more than 24 MiB of scratch (at d = 64 every split plan on a 148-SM B200 fits; at
 *     d = 128 split plans of more than about 94 CTAs do not -- use attn_fwd_ws for those).
 *     Shapes that need no split mode never touch the array and are never rejected.
 *   - The first call on a device looks up the array's device address with that device
 *     current; make that first call before any stream capture.
 *   - Every call shares the one array and it keeps the previous call's contents; each call
 *     clears the part that must start at zero (a memset on `stream`).  Calls whose execution
 *     overlaps on the GPU (different streams, different host threads, no ordering between
 *     them) race on the array and may return wrong results: order them.
 */
int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Nq, int Nk, int d, float scale, int causal, int dtype,
                     attn_stream_t stream);

/*
 * attn_fwd_stall_test -- test hook for the failure path; not for production use.
 *
 * Enqueues attn_fwd_ws (same arguments) with one internal wait pointed at a barrier that
 * nothing ever arrives on, so that the bounded wait runs out after about one second:
 *   stall_site 1: softmax warpgroup 0, before its first score tile;
 *              2: the MMA warp, before its first MMA;
 *              3: the Q/K TMA warp, before its first load;
 *              4: softmax warpgroup 0, before the split-piece rendezvous (split mode only;
 *                 the shapes for which attn_plan reports split = 1).
 * The kernel records 0x8000000A in the device status word, every role leaves its loop, the
 * issued loads and MMAs are waited for, tensor memory is freed and the kernel returns;
 * attn_get_device_status() then reports ATTN_ERR_DEVICE_TIMEOUT and the CUDA context stays
 * usable.  o / lse hold no meaningful result; a split-mode workspace must be zero-filled
 * again afterwards.  Returns ATTN_ERR_SHAPE for a stall_site outside 1..4, otherwise the
 * codes of attn_fwd_ws.  Nothing here faults or traps the GPU.
 */
int attn_fwd_stall_test(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int Nq, int Nk, int d, float scale, int causal, int dtype,
                        void* workspace, size_t workspace_bytes, int stall_site,
                        attn_stream_t stream);

/*
 * attn_fwd_host -- the same forward, end to end from host memory.
 *
 * Host->device copies of q_host, k_host, v_host into the caller's device buffers q_dev,
 * k_dev, v_dev; the forward on them into o_dev / lse_dev; device->host copies of o_dev into
 * o_host and (when both lse pointers are non-NULL) lse_dev into lse_host.  The whole call is
 * ordered after the work already enqueued on `stream`, and work enqueued on `stream`
 * afterwards runs after it; the caller synchronises `stream` before reading o_host.  Host
 * buffers must be pinned (cudaHostAlloc / cudaHostRegister) for the copies to be
 * asynchronous.
 *
 * Problems with at least 4 MB of input that run in unit mode are pipelined: the (batch,
 * head) slices are cut into up to 8 contiguous chunks, and chunk c's copies in, forward and
 * copies out run on three streams the library creates once per device (with events chaining
 * them), so copies of one chunk overlap the compute and the opposite-direction copies of
 * the others.  The result is bit-for-bit that of attn_fwd.  Calls from several host threads
 * share those streams and are serialised by a lock while they enqueue.  Smaller problems,
 * and problems that take split mode from `workspace`, run as one copy-in / forward /
 * copy-out sequence on `stream`.
 *
 * Argument rules and error codes are those of attn_fwd; every host and device pointer
 * except the lse pair must be non-NULL.  workspace / workspace_bytes are optional (NULL, 0)
 * and act as in attn_fwd_ws.  Nothing is allocated per call.  Argument errors are found
 * before anything is enqueued.  If a CUDA call fails after some copies were enqueued, the
 * call still orders `stream` after everything it enqueued before returning the error, so a
 * synchronisation of `stream` is enough before the host buffers are freed or reused; the
 * outputs are then invalid.
 */
int attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                  float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                  float* lse_dev, void* workspace, size_t workspace_bytes, int B, int H, int Nq,
                  int Nk, int d, float scale, int causal, int dtype, attn_stream_t stream);

/*
 * attn_bwd -- gradients of the forward: dq, dk, dv for an output gradient dout.
 *
 * The backward pass of training, with the softmax recomputed from the statistics the forward
 * saved instead of being stored ("YOLOv12推理速度翻倍秘诀：Flash Attention加持" (0539edu.com),
 * section 1; YOLO11 x FlashAttention-2 (kwkr.cn), sections 2.3 and 4.3).  For each (batch,
 * head), with S = scale * Q K^T (masked as in attn_fwd) and P = exp(S - lse):
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),  dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 *   q, k, v    the forward's inputs (layouts of attn_fwd).
 *   o, lse     the forward's outputs for exactly these inputs, scale and causal flag: o
 *              [B, H, Nq, d] in `dtype`, lse [B, H, Nq] float32 (lse is required here).
 *   dout       dL/dO, [B, H, Nq, d] in `dtype`.
 *   dq, dk, dv outputs, shaped and typed like q, k, v (fully overwritten; rows a causal mask
 *              hides from every query get zero gradients).
 *   workspace  caller-owned device memory of at least attn_bwd_workspace_size bytes,
 *              16-byte aligned; contents need not be initialised and are left undefined.
 *
 * Three kernels run in order on `stream`: a row pass (D = rowsum(dO * O), lse in base 2,
 * zeroing an fp32 dQ accumulator in the workspace), the main pass (one CTA per 128-key tile
 * and (batch, head): recomputed P, dS, and dK, dV accumulated in tensor memory, dQ added into
 * the accumulator with atomic vector adds) and a pass converting dQ to `dtype`.  Because the
 * dQ additions from different key tiles land in any order, dq can differ in the last bits
 * between calls; dk and dv are deterministic.
 *
 * Errors: as attn_fwd for q, k, v, o, lse (NULL lse is ATTN_ERR_NULL) and for dout, dq, dk, dv
 * (NULL, 16-byte alignment); ATTN_ERR_WORKSPACE for the workspace.  Nothing is enqueued on an
 * argument error.  Nothing is allocated per call.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d,
             float scale, int causal, int dtype, void* workspace, size_t workspace_bytes,
             attn_stream_t stream);

/* Workspace bytes attn_bwd needs for these sizes (host arithmetic only; no GPU needed). */
int attn_bwd_workspace_size(int B, int H, int Nq, int Nk, int d, size_t* bytes);

/*
 * attn_qkv_proj -- the qkv projection of the attention block, written in the attention layout.
 *
 * [q | k | v] = x W_qkv^T (+ b_qkv) for x [B, N, C] with C = H * d, W_qkv [3 C, C] (an
 * nn.Linear(C, 3 C) weight) and b_qkv [3 C] float32 or NULL (the page's qkv Linear has no
 * bias).  Column c of the product goes to tensor c / C (q, k, v), head (c % C) / d, element
 * c % d -- the reshape to [B, N, 3, H, d], unbind and transpose of the YOLO11 x
 * FlashAttention-2 page (kwkr.cn), section 2.2 -- so q, k, v come out as [B, H, N, d]
 * contiguous, ready for attn_fwd, with no reshape pass.  One tcgen05 GEMM (fp32 accumulation,
 * one rounding to `dtype`).  x, W_qkv, q, k, v 16-byte aligned; b_qkv 4-byte aligned.  Errors:
 * ATTN_ERR_NULL, ATTN_ERR_DTYPE, ATTN_ERR_HEAD_DIM (d not 64 / 128), ATTN_ERR_SHAPE,
 * ATTN_ERR_ALIGN, ATTN_ERR_ARCH, ATTN_ERR_CUDA; nothing is enqueued on an argument error.
 */
int attn_qkv_proj(const void* x, const void* w_qkv, const float* b_qkv, void* q, void* k,
                  void* v, int B, int N, int H, int d, int dtype, attn_stream_t stream);

/*
 * attn_out_proj -- the output projection, reading the attention output in its own layout.
 *
 * y = o' W_o^T (+ b_o) where o' [B, N, H d] is o [B, H, N, d] transposed back (the page's
 * o.transpose(1, 2).reshape(B, N, C)), W_o [C_out, H d] and b_o [C_out] float32 or NULL; y is
 * [B, N, C_out] in `dtype`.  The GEMM's first operand is loaded from o through a 4-D tensor
 * map, so the transpose is never written out.  C_out must be a multiple of 8.  o, W_o, y
 * 16-byte aligned.  Errors as attn_qkv_proj.
 */
int attn_out_proj(const void* o, const void* w_o, const float* b_o, void* y, int B, int N, int H,
                  int d, int C_out, int dtype, attn_stream_t stream);

/*
 * attn_block_fwd -- the whole attention block: attn_qkv_proj, attn_fwd (Nq = Nk = N), then
 * attn_out_proj, enqueued in that order on `stream` after every argument has been checked.
 * q, k, v, o [B, H, N, d] and lse [B, H, N] (or NULL) are caller-owned intermediates and keep
 * their values.  Errors as the three calls.
 */
int attn_block_fwd(const void* x, const void* w_qkv, const float* b_qkv, const void* w_o,
                   const float* b_o, void* q, void* k, void* v, void* o, float* lse, void* y,
                   int B, int N, int H, int d, int C_out, float scale, int causal, int dtype,
                   attn_stream_t stream);

/*
 * attn_plan -- the launch geometry attn_fwd would use for these sizes on a GPU with
 * `num_sms` SMs (pure host arithmetic; needs no GPU).  Returns ATTN_ERR_SHAPE /
 * ATTN_ERR_HEAD_DIM / ATTN_ERR_NULL on bad arguments, else ATTN_OK with *out filled.
 */
int attn_plan(int B, int H, int Nq, int Nk, int d, int causal, int num_sms, attn_plan_t* out);

/*
 * attn_get_device_status -- synchronises `stream`, then reads and clears the device status
 * word the kernels write when a bounded internal wait gives up (about one second).  Returns
 * ATTN_OK when healthy, ATTN_ERR_DEVICE_TIMEOUT when a kernel timed out (the result of that
 * call is invalid; the CUDA context stays usable), ATTN_ERR_CUDA if the synchronisation or
 * the read fails.  When `detail` is non-NULL it receives the raw status word (0 = healthy;
 * else 0x80000000 | wait site).
 */
int attn_get_device_status(attn_stream_t stream, unsigned int* detail);

/* Static English message for a status code; never NULL. */
const char* attn_strerror(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_SM100_ATTN_H_ */
