/*
 * spa2.h -- C ABI of libspa2.so: hybrid Top-k + Top-p block-sparse attention
 * (SpargeAttention2) on NVIDIA B200 (sm_100a).
 *
 * The operations are those of arXiv 2602.13515, "SpargeAttention2: Trainable
 * Sparse Attention via Hybrid Top-k+Top-p Masking and Distillation
 * Fine-Tuning", as summarised on
 *   - paper.rainbus.top (SpargeAttention2 summary), sections 前置知识
 *     (sparse / Top-k / Top-p / block-sparse attention), 方法步骤详情 (method
 *     steps 1-4) and 技术新颖性 (the union formula);
 *   - gist.science (same title), section 2A "Hybrid Top-k + Top-p Masking"
 *     and 2C "Efficient Kernel Implementation";
 *   - chatpaper.ai abstract ("efficient trainable sparse attention
 *     implementation": forward and backward).
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * Tensors. Q, K, V, O, dO, dQ, dK, dV are contiguous [B, H, N, d] bf16 in
 *   device memory, 16-byte aligned. LSE is [B, H, N] fp32 (natural log of the
 *   row sum of exp(scaled logits)). Block counts: T_m = ceil(N / bq),
 *   T_n = ceil(N / bkv); the last block of a ragged N is partial.
 * Supported set. d in {64, 128}; bq in {64, 128, 256}; bkv in {64, 128};
 *   1 <= N <= 131072; B, H >= 1 with B*H <= 65535; 0 <= k_frac <= 1,
 *   0 <= p_frac <= 1. (bq, bkv) = (128, 64) is the method's setting and the
 *   fastest path; the other sizes run the same attention kernels on tiles of
 *   128 query rows x 64 key rows through tile lists built at the start of the
 *   forward / backward call (per-layer block sizes: paper.rainbus.top,
 *   独立分析的弱点). Anything else returns
 *   SPA2_ERR_UNSUPPORTED (or SPA2_ERR_INVALID_ARG for nonsense such as a null
 *   pointer or a negative size) and launches nothing.
 * Ownership. The caller allocates and owns every buffer, including the
 *   workspace `ws` (size from spa2_workspace_bytes, 256-byte aligned). The
 *   library never allocates or frees device memory and keeps no pointer
 *   after a call returns.
 * Streams. All work is enqueued asynchronously on `stream` (NULL = the
 *   legacy default stream); a call returns once its kernels are enqueued.
 * Errors. Argument errors are returned synchronously before anything is
 *   launched. A failed launch returns SPA2_ERR_CUDA. Faults detected on the
 *   device (a bounded wait that ran out, an index outside its buffer) are
 *   recorded in the status word (the first 4 bytes of `ws`, cleared at the
 *   start of every call) and read back by spa2_stream_status. The library
 *   never aborts, asserts or traps.
 */
#ifndef SPA2_H
#define SPA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SPA2_API __attribute__((visibility("default")))
#else
#define SPA2_API
#endif

typedef struct CUstream_st* spa2_stream_t; /* identical to cudaStream_t */

typedef enum {
  SPA2_OK = 0,
  SPA2_ERR_INVALID_ARG = 1,    /* null pointer, negative size, misaligned pointer */
  SPA2_ERR_UNSUPPORTED = 2,    /* valid but outside the supported set above */
  SPA2_ERR_CUDA = 3,           /* a CUDA runtime / driver call failed */
  SPA2_ERR_DEVICE_TIMEOUT = 4, /* a device-side bounded wait ran out */
  SPA2_ERR_WORKSPACE = 5,      /* ws is NULL or smaller than spa2_workspace_bytes */
  SPA2_ERR_DEVICE_BOUNDS = 6, /* a device-side index check failed (bad mask) */
  SPA2_ERR_RANGE = 7           /* an input value outside the supported range (|V| > 65504) */
} spa2_status;

/*
 * Block mask in compressed form. All pointers are device pointers owned by
 * the caller. Kept ids of a row (column) are listed in ascending order; only
 * the first row_cnt (col_cnt) entries of a row (column) are meaningful.
 *   row_cnt [B, H, T_m]       int32  kept kv-blocks per q-block (>= 1)
 *   row_idx [B, H, T_m, T_n]  int32  kept kv-block ids of each q-block (CSR)
 *   col_cnt [B, H, T_n]       int32  q-blocks keeping each kv-block
 *   col_idx [B, H, T_n, T_m]  int32  those q-block ids (CSC)
 *   pbar    [B, H, T_m, T_n]  fp32   pooled attention P-bar, or NULL
 *   bitmap  [B, H, T_m, T_n]  uint8  1 = kept, or NULL
 * spa2_sparse_attn_fwd reads row_cnt/row_idx; spa2_sparse_attn_bwd reads
 * both; the mask builders write all non-NULL fields (col_* may be NULL when no
 * backward pass will follow).
 */
typedef struct {
  int32_t* row_cnt;
  int32_t* row_idx;
  int32_t* col_cnt;
  int32_t* col_idx;
  float* pbar;
  uint8_t* bitmap;
} spa2_mask;

enum { SPA2_OP_MASK = 0, SPA2_OP_FWD = 1, SPA2_OP_BWD = 2, SPA2_OP_SELECT = 3 };

/* Element type of the gradient outputs of spa2_sparse_attn_bwd. */
enum { SPA2_DTYPE_BF16 = 0, SPA2_DTYPE_F32 = 1 };

/* ABI version of this header (bumped on any incompatible change). */
#define SPA2_ABI_VERSION 1
SPA2_API int spa2_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
SPA2_API const char* spa2_status_string(spa2_status s);

/*
 * Workspace bytes needed by `op` (SPA2_OP_*) for this shape; 0 for an
 * unsupported shape. For SPA2_OP_SELECT the arguments are read as
 * (B, H, T_m, T_n) = (B, H, N, d) and bq, bkv are ignored. Every workspace
 * starts with the 256-byte status block.
 */
SPA2_API size_t spa2_workspace_bytes(int op, int B, int H, int N, int d, int bq, int bkv);

/*
 * Steps 1-3 of the method (paper.rainbus.top, 方法步骤详情, steps 1-3):
 *   1. partition Q into T_m blocks of bq rows, K into T_n blocks of bkv rows;
 *   2. pool each block to its mean row (fp32) and form the pooled attention
 *      P-bar = softmax(pool(Q) pool(K)^T / sqrt(d)), row by row;
 *   3. keep block j of row i iff j is in Top-k(P-bar_i, k_frac) or in
 *      Top-p(P-bar_i, p_frac) (union; 技术新颖性 formula).
 * Selection rule (exact, deterministic): rank the row by (P-bar descending,
 * block id ascending); K = clamp(floor(k_frac * T_n + 0.5), 1, T_n) in double;
 * Top-p keeps rank r while floor(2^32 * mass of ranks < r) < floor(2^32 *
 * p_frac), masses quantised per block as floor(2^32 * P-bar_j) (the first
 * prefix whose mass reaches p, sink row example of 研究动机); the union is the
 * first max(K, R) ranks. Writes every non-NULL field of *out.
 *   q, k : [B, H, N, d] bf16 device pointers (read only)
 *   out  : host pointer to a spa2_mask of device pointers (see above)
 *   ws   : device workspace of spa2_workspace_bytes(SPA2_OP_MASK, ...) bytes
 */
SPA2_API spa2_status spa2_block_mask(const void* q, const void* k, int B, int H, int N, int d, int bq, int bkv,
                            float k_frac, float p_frac, const spa2_mask* out, void* ws, size_t ws_bytes,
                            spa2_stream_t stream);

/*
 * spa2_block_mask without a caller workspace. The method has no counterpart
 * of this entry point: it exists for callers that cannot hand the library a
 * workspace at call time, such as a plain C host program on a fixed memory
 * plan with no device allocator of its own, or a step loop that must not call
 * cudaMalloc (which synchronises the whole device) between kernels.
 * Computes exactly what spa2_block_mask computes, with the same kernels.
 *   scratch: one file-scope device array of SPA2_NOALLOC_MASK_SCRATCH_BYTES
 *            per device, part of the library's image; nothing is allocated
 *            by the call. A shape whose mask workspace
 *            (spa2_workspace_bytes(SPA2_OP_MASK, ...)) exceeds that size is
 *            refused with SPA2_ERR_WORKSPACE before any launch.
 *   setup:   the first call on a device (with that device current) looks the
 *            array's address up once and caches it; make that first call
 *            before any stream capture begins on that device. A
 *            cudaDeviceReset unloads the library's device image, and with it
 *            the array: calls on that device after a reset are not supported
 *            (the cached address is stale).
 *   status:  NULL, or a 4-byte-aligned device int the caller owns; the call
 *            copies the device-side status word there (stream-ordered). Read
 *            it with spa2_stream_status(status, stream). With status == NULL
 *            device-side errors of the call (a timed-out wait, a failed bounds
 *            check) are discarded: nothing reports them.
 *   races:   all calls on one device share the array. Calls issued one after
 *            another on one stream are safe; calls whose executions overlap
 *            (other streams, other host threads) race and give wrong masks.
 * Arguments and outputs otherwise as spa2_block_mask.
 */
#define SPA2_NOALLOC_MASK_SCRATCH_BYTES (64u << 20) /* 64 MiB */
SPA2_API spa2_status spa2_block_mask_noalloc(const void* q, const void* k, int B, int H, int N, int d, int bq,
                                    int bkv, float k_frac, float p_frac, const spa2_mask* out, int* status,
                                    spa2_stream_t stream);

/*
 * Step 3 alone on a caller-given P-bar (parity checks of the selection rule,
 * and masks computed elsewhere). Same rule and outputs as spa2_block_mask;
 * out->pbar is ignored. pbar entries must be finite and in [0, 1]; T_n <= 2048.
 *   pbar : [B, H, T_m, T_n] fp32 device pointer
 *   ws   : spa2_workspace_bytes(SPA2_OP_SELECT, B, H, T_m, T_n, 0, 0) bytes
 */
SPA2_API spa2_status spa2_select_blocks(const float* pbar, int B, int H, int Tm, int Tn, float k_frac, float p_frac,
                               const spa2_mask* out, void* ws, size_t ws_bytes, spa2_stream_t stream);

/*
 * Step 4 forward (paper.rainbus.top, 方法步骤详情 step 4 and 前置知识 "稀疏注意力",
 * "块稀疏注意力"; gist.science 2C): for every q-block i and every kept kv-block j
 * of row i, S_ij = Q_i K_j^T * softmax_scale, online softmax, O_i += P_ij V_j;
 * masked (i, j) tiles are skipped entirely. No causal mask.
 * Precision: S = Q K^T takes bf16 operands; P V runs with fp16 operands (P in
 * [0, 256] and an fp16 copy of V made in the workspace, exact for bf16 V with
 * |V| <= 65504; larger values are clamped and reported as SPA2_ERR_RANGE),
 * fp32 accumulation throughout.
 *   q, k, v       : [B, H, N, d] bf16 device pointers (read only)
 *   mask          : host pointer to a spa2_mask; row_cnt/row_idx are read
 *   softmax_scale : logit scale; 0 means 1/sqrt(d)
 *   o             : [B, H, N, d] bf16 device output, O rounded to nearest
 *   o_lo          : optional [B, H, N, d] bf16 device output, the residual
 *                   bf16(O - o) of the fp32 O (o + o_lo carries ~16 mantissa
 *                   bits); pass it to the backward for an accurate
 *                   D = rowsum(dO * O). NULL skips it.
 *   lse           : [B, H, N] fp32 device output (natural-log LSE)
 *   ws            : spa2_workspace_bytes(SPA2_OP_FWD, ...) bytes (fp16 copy of
 *                   V, and the tile lists for sizes other than (128, 64))
 */
SPA2_API spa2_status spa2_sparse_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                          int bq, int bkv, const spa2_mask* mask, float softmax_scale, void* o,
                                          void* o_lo, float* lse, void* ws, size_t ws_bytes, spa2_stream_t stream);

/*
 * Step 4 backward through the same block mask (the trainable part;
 * chatpaper.ai abstract (ii)): with P = exp(S - LSE) on kept tiles,
 *   dV_j = sum_i P_ij^T dO_i,  dP_ij = dO_i V_j^T,  D_i = rowsum(dO_i * O_i),
 *   dS_ij = P_ij * (dP_ij - D_i),  dQ_i = sum_j dS_ij K_j * scale,
 *   dK_j = sum_i dS_ij^T Q_i * scale.
 * The mask is held constant (no gradient through pooling or selection).
 * Precision: the dK/dV pass runs every product on fp16 values of Q, K, V and
 * dO (bf16 -> fp16 is exact for magnitudes in [2^-14, 65504]; smaller ones
 * round to fp16 subnormals, absolute error <= 2^-25): S = Q K^T, dP = dO V^T,
 * and P (in [0, 1]) and dS enter dV = P^T dO and dK = dS^T Q as fp16. The dQ
 * pass recomputes S and dP from the bf16 inputs, and dS enters dQ = dS K as
 * a hi + lo pair of bf16 values (about 16 significant bits). Accumulation is
 * fp32 throughout and D uses o + o_lo when o_lo is given. Q, K, V or dO of
 * magnitude > 65504 is clamped for the fp16 values and reported as
 * SPA2_ERR_RANGE.
 * dK and dV are accumulated per kv-block (CSC column), dQ per q-block (CSR
 * row, recomputing S and dP), so no output is accumulated atomically and the
 * results are deterministic.
 *   q, k, v, o, dout : [B, H, N, d] bf16 device pointers (read only); o, o_lo
 *                      and lse are the forward outputs for the same mask
 *   o_lo             : optional [B, H, N, d] bf16 residual of O (or NULL)
 *   lse              : [B, H, N] fp32 device pointer
 *   mask             : host pointer to a spa2_mask; row_cnt/row_idx and
 *                      col_cnt/col_idx are read
 *   dq, dk, dv       : [B, H, N, d] device outputs of type grad_dtype
 *   grad_dtype       : SPA2_DTYPE_BF16 or SPA2_DTYPE_F32
 *   ws               : spa2_workspace_bytes(SPA2_OP_BWD, ...) bytes (holds D,
 *                      fp16 copies of dO and Q, the order in which the dK/dV
 *                      pass takes its kv columns, and the tile lists for sizes
 *                      other than (128, 64))
 */
SPA2_API spa2_status spa2_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                                          const void* o_lo, const float* lse, const void* dout, int B, int H, int N,
                                          int d, int bq, int bkv, const spa2_mask* mask, float softmax_scale,
                                          void* dq, void* dk, void* dv, int grad_dtype, void* ws, size_t ws_bytes,
                                          spa2_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the status word at the start
 * of `ws`. Returns SPA2_OK, the first device-side error recorded since the
 * word was last cleared, or SPA2_ERR_CUDA if the stream itself failed.
 */
SPA2_API spa2_status spa2_stream_status(void* ws, spa2_stream_t stream);

/*
 * Fault-path testing. Sets the time limit, in nanoseconds, of every bounded
 * device-side wait launched afterwards by this process (default 2e9 = 2 s;
 * limit <= 0 restores the default). Returns SPA2_OK.
 */
SPA2_API spa2_status spa2_debug_set_wait_limit_ns(long long limit);

/*
 * Fault-path testing. Launches one CTA that waits on an mbarrier nothing
 * arrives on, bounded by the current wait limit; the wait runs out, the
 * kernel records SPA2_ERR_DEVICE_TIMEOUT in the status word of `ws` (>= 256
 * bytes) and returns normally, leaving the context usable.
 */
SPA2_API spa2_status spa2_debug_timeout_probe(void* ws, size_t ws_bytes, spa2_stream_t stream);

/*
 * Per-kernel timing, a measurement aid with no counterpart in the method.
 * While timing is on, every kernel the library launches is bracketed by two
 * CUDA events recorded on its launch stream (this adds a few microseconds of
 * event records per call and nothing else; results are unchanged). Events are
 * created on demand (cudaEventCreate; no device memory) and recycled.
 *   spa2_timing_enable(on)  on != 0 starts recording, 0 stops; returns SPA2_OK.
 *   spa2_kernel_count()     number of kernel kinds (ids 0 .. count-1).
 *   spa2_kernel_name(id)    static name of kernel kind `id` ("unknown" if out of range).
 *   spa2_timing_read(n, launches, total_ms)
 *                           waits for every event recorded since the last read,
 *                           writes for ids 0 .. n-1 the number of launches and
 *                           their summed event time in milliseconds (host arrays
 *                           of n entries), then forgets the recorded launches.
 *                           SPA2_ERR_CUDA if an event could not be read (e.g.
 *                           it was recorded during stream capture);
 *                           SPA2_ERR_INVALID_ARG for n < 0 or NULL arrays.
 */
SPA2_API spa2_status spa2_timing_enable(int on);
SPA2_API int spa2_kernel_count(void);
SPA2_API const char* spa2_kernel_name(int kernel_id);
SPA2_API spa2_status spa2_timing_read(int n, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* SPA2_H */
