/*
 * h3attn — quantized dense self-attention for the H3 video-diffusion block,
 * native to NVIDIA B200 (sm_100a).  C ABI of libh3attn.so.
 *
 * The operation is the dense Sage-compatible attention of "H3 Performance
 * Roadmap", Phase 4: Dense Sage-Compatible Attention: it consumes strided BSHD
 * Q/K/V views directly, keeps the SageAttention 2.2.0 numerical policy
 * (per-warp INT8 Q/K with K smoothing, FP8 V, FP32 accumulation) and writes
 * token-major output that the out-projection reads without a copy.  Its
 * numerical checkpoints are those of "Phase 2B Aligned Numerical Prototype",
 * Exactness (INT32-to-FP32 QK scores, per-epoch online-softmax m and d, FP8
 * E4M3 probability words, FP32 RO, final reciprocal, BF16 output).
 *
 * Policy implemented (D = 128; all divisions and products correctly rounded):
 *   km[b,h,c]   = mean over the Tkv keys of K[b,:,h,c]  (FP64 sums, FP32 result)
 *   Q groups    : 32 tokens per (b,h); sq = amax/127; q8 = clamp(rne(x*(127/amax)), +-127)
 *   K groups    : 64 tokens per (b,h), on K - km, same rule -> k8, sk
 *   V channels  : sv = amax_c/448;  v8 = e4m3_rne_satfinite(v * (448/amax_c))
 *   scores      : acc = sum_c q8*k8 (exact INT32);  t = float(acc) * ((sq*sk) * c),
 *                 c = float(softmax_scale * log2(e));  keys >= Tkv masked
 *   per 128-key tile: m' = max(m, max t); alpha = 2^(m - m'); p = 2^(t - m');
 *                 d = d*alpha + sum p;  p8 = e4m3(448*p);  RO = RO*alpha + p8 x v8
 *   out         = bf16((RO * (1/d)) * (sv/448))
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, except the
 *     host views of h3attn_forward_host.  The library never allocates or frees
 *     device memory and never synchronises except in h3attn_check_status (and
 *     h3attn_forward_host_check_status); h3attn_forward_host creates two copy
 *     streams and eight events per call and releases them before it returns, and
 *     h3attn_forward_static uses its own static device array.  Other than that
 *     array, the library keeps no state between calls beyond per-device caches of
 *     kernel attributes.
 *   - Element strides are in BF16 elements; the channel (d) stride is 1.
 *     Base pointers must be 16-byte aligned and strides multiples of 8
 *     elements (16-byte vector loads); the workspace must be 256-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously.  Argument errors are returned
 *     synchronously and nothing is enqueued.  Errors found on the device (a
 *     bounded wait that expired) are recorded in the workspace's status word
 *     and returned by h3attn_check_status.  The status word is sticky: the
 *     first failure of any call made on a workspace stays recorded, through
 *     later calls on the same workspace, until h3attn_check_status reads and
 *     clears it.  (The quantize pass initialises the status block only on a
 *     workspace that does not hold its 64-bit marker yet, i.e. a new one.)
 *   - Inputs are assumed finite; NaN or Inf inputs give undefined output.
 *   - Output must not overlap the inputs or the workspace.
 */
#ifndef H3ATTN_H_
#define H3ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define H3ATTN_VERSION 1
#define H3ATTN_HEAD_DIM 128
#define H3ATTN_Q_GROUP 32    /* Q tokens per INT8 scale ("per-warp" Q quantization) */
#define H3ATTN_K_GROUP 64    /* K tokens per INT8 scale (one K64 epoch) */
#define H3ATTN_TILE 128      /* Q rows and keys per tile of the attention kernel */

typedef enum {
  H3ATTN_OK = 0,
  H3ATTN_ERR_INVALID_ARG = 1,  /* null pointer, size < 1, bad index */
  H3ATTN_ERR_UNSUPPORTED = 2,  /* D != 128, or the current device is not sm_100 */
  H3ATTN_ERR_ALIGNMENT = 3,    /* pointer or stride violates the alignment rules */
  H3ATTN_ERR_WORKSPACE = 4,    /* workspace null, misaligned or smaller than needed */
  H3ATTN_ERR_CUDA = 5,         /* a CUDA runtime or driver call failed */
  H3ATTN_ERR_TIMEOUT = 6       /* a device-side bounded wait expired (read via check_status) */
} h3attn_status;

/* A read-only BF16 tensor viewed as [B, T, H, D]; strides in elements, d stride 1. */
typedef struct {
  const void* data;
  int64_t stride_b, stride_t, stride_h;
} h3attn_bf16_view;

/* A writable BF16 tensor viewed as [B, T, H, D]; strides in elements, d stride 1.
 * The out-projection layout [B, T, H*D] is stride_b = T*H*D, stride_t = H*D, stride_h = D. */
typedef struct {
  void* data;
  int64_t stride_b, stride_t, stride_h;
} h3attn_bf16_out;

/* Workspace fields, in the order h3attn_workspace_layout reports their byte offsets. */
enum {
  H3ATTN_WS_STATUS = 0, /* status block, 256 bytes: int32 code, detail, block, 64-bit marker */
  H3ATTN_WS_Q8,         /* INT8 Q words held as BF16 values (exact), [B, H, Tq_pad, 128];
                           Tq_pad = ceil(Tq/128)*128, rows >= Tq are 0 */
  H3ATTN_WS_K8,         /* INT8 K words held as BF16 values, [B, H, Tkv_pad, 128];
                           Tkv_pad = ceil(Tkv/128)*128, rows >= Tkv are 0 */
  H3ATTN_WS_V8T,        /* e4m3  [B, H, 128, Tkv_pad]  V transposed (channel-major), columns >= Tkv are 0 */
  H3ATTN_WS_SQ,         /* f32   [B, H, Tq_pad/32]     Q group scales (0 for groups past Tq) */
  H3ATTN_WS_SK,         /* f32   [B, H, Tkv_pad/64]    K group scales (0 for groups past Tkv) */
  H3ATTN_WS_KM,         /* f32   [B, H, 128]           K channel means */
  H3ATTN_WS_SV,         /* f32   [B, H, 128]           V channel scales amax/448 */
  H3ATTN_WS_KSUM,       /* f64   [B, H, ceil(Tkv/64), 128]  scratch: per-chunk K sums */
  H3ATTN_WS_VMAX,       /* f32   [B, H, ceil(Tkv/64), 128]  scratch: per-chunk V absmax */
  H3ATTN_WS_END,        /* total bytes */
  H3ATTN_WS_NFIELDS
};

/* Bytes of workspace needed for (B, Tq, Tkv, H, D); 0 if the sizes are invalid. */
size_t h3attn_workspace_bytes(int B, int Tq, int Tkv, int H, int D);

/* Byte offsets of every workspace field (see the enum above) into offsets[H3ATTN_WS_NFIELDS]. */
h3attn_status h3attn_workspace_layout(int B, int Tq, int Tkv, int H, int D,
                                      int64_t offsets[H3ATTN_WS_NFIELDS]);

/* K smoothing, Q/K INT8 and V FP8 quantization ("H3 Performance Roadmap", the
 * Sage2 decomposition: K smoothing, Q/K INT8 quantization, V transpose and FP8
 * quantization).  Reads q (Tq tokens) and k, v (Tkv tokens); writes every
 * field of the workspace (the status block only when it is new, see the
 * conventions above).  Three kernels (per-chunk
 * statistics, their ordered reduction, one quantize pass), or one kernel doing
 * all three per (b, h) when max(Tq, Tkv) is at most 512 tokens; both give the
 * same words. */
h3attn_status h3attn_quantize_qkv(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                  const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                  void* ws, size_t ws_bytes, void* stream);

/* The fused attention mainloop on a workspace filled by h3attn_quantize_qkv with the
 * same sizes: QK^T of the INT8 words on the tensor cores into tensor memory (BF16
 * operands holding the integers, FP32 accumulation: exact, since every product and
 * partial sum is an integer below 2^24), FP32 online softmax, FP8 P, FP8 PV with FP32
 * accumulation, final reciprocal, BF16 store of rows < Tq into `out`.
 * softmax_scale is usually 1/sqrt(D). */
h3attn_status h3attn_attend(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H, int D,
                            float softmax_scale, const h3attn_bf16_out* out, void* stream);

/* Quantize + attend for self-attention (Tq == Tkv == T). */
h3attn_status h3attn_forward(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                             const h3attn_bf16_view* v, int B, int T, int H, int D,
                             float softmax_scale, const h3attn_bf16_out* out,
                             void* ws, size_t ws_bytes, void* stream);

/* Quantize + attend with separate query and key lengths. */
h3attn_status h3attn_forward_ex(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                float softmax_scale, const h3attn_bf16_out* out,
                                void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns the device status recorded in the workspace
 * (H3ATTN_OK or H3ATTN_ERR_TIMEOUT: the first failure of any call on this workspace
 * since the last check) and clears it.  ws must be at least 256 bytes. */
h3attn_status h3attn_check_status(void* ws, void* stream);

/* Parity export: the exact INT32 QK^T tile of (b, h, Q tile qt, key tile kt) as
 * computed by the same tensor-core path the attention kernel uses, written as
 * 128 x 128 row-major int32 to the device buffer out_dev (caller-owned, 16-byte
 * aligned; rows or keys past Tq/Tkv hold the products of the zero padding).  ws must
 * hold a quantize pass of the same sizes.  H3ATTN_ERR_INVALID_ARG for indices out of
 * range or a null out_dev, H3ATTN_ERR_ALIGNMENT for a misaligned one.  The INT32
 * score checkpoint of "Phase 2B Aligned Numerical Prototype", Exactness. */
h3attn_status h3attn_debug_qk_scores(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H,
                                     int D, int b, int h, int qt, int kt, int32_t* out_dev,
                                     void* stream);

/* Device bytes h3attn_forward_host needs for these sizes and heads_per_group (two
 * slots of staged Q, K, V and output plus a workspace for heads_per_group heads);
 * 0 for invalid sizes or heads_per_group outside [1, H]. */
size_t h3attn_forward_host_bytes(int B, int Tq, int Tkv, int H, int D, int heads_per_group);

/* The head groups of h3attn_forward_host(..., H, ..., heads_per_group): heads_per_group
 * heads each, except that when H > 2 * heads_per_group (and heads_per_group >= 2) the
 * first and the last group take heads_per_group / 2 heads.  Writes the first head of
 * each group and then H to group_start[0 .. n] (n + 1 ints; NULL to only count, at most
 * H + 1 entries are written) and returns the number of groups n; 0 for heads_per_group
 * outside [1, H] or H outside [1, 4096]. */
int h3attn_forward_host_groups(int H, int heads_per_group, int* group_start);

/* Forward pass (as h3attn_forward_ex) from HOST input views to a HOST output view, for
 * callers whose activations are not resident on the device.  The heads are processed in
 * the groups of h3attn_forward_host_groups: group g is uploaded on an internal stream,
 * computed on `stream`, and downloaded on a second internal stream, so the upload of
 * group g+1 and the download of group g-1 overlap the kernels of group g.  Only the
 * first group's upload and the last group's download stand alone, which is why those two
 * groups are the smaller ones.  Heads are independent
 * problems (every statistic, scale and softmax is per (b, h)), so the result is bit for
 * bit that of one h3attn_forward_ex call on all heads.
 *   q, k, v, out: host views with the device views' rules (16-byte aligned data, strides
 *     in elements, multiples of 8, channel stride 1); page-locked memory for the copies
 *     to overlap.  The caller keeps them alive and unmodified until `stream` reaches the
 *     end of the call (every copy of the call is ordered before that point).
 *   dev_buf: device memory of h3attn_forward_host_bytes(...) bytes, 1024-byte aligned,
 *     owned by the caller; holds the staging and the per-slot workspaces.
 *   H: at most 4096 (H3ATTN_ERR_INVALID_ARG beyond).
 * Asynchronous on `stream`; creates its two copy streams and eight events per call and
 * releases them before returning (the runtime frees them once their work is done).
 * Device-side status: h3attn_forward_host_check_status.  The zero-copy layout of
 * "H3 Performance Roadmap", Phase 4 item 5 (token-major in and out) applies to the host
 * views the same way. */
h3attn_status h3attn_forward_host(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                  const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                  float softmax_scale, const h3attn_bf16_out* out, int heads_per_group,
                                  void* dev_buf, size_t dev_bytes, void* stream);

/* h3attn_check_status for the workspaces inside an h3attn_forward_host buffer: the
 * first non-OK status of the slots the calls used (each is read and cleared).  The
 * status words are sticky, so a timeout in any head group of any call since the last
 * check is reported, not only one in the last two groups. */
h3attn_status h3attn_forward_host_check_status(void* dev_buf, int B, int Tq, int Tkv, int H, int D,
                                               int heads_per_group, void* stream);

/* Failure-path test hook of the host pipeline: h3attn_forward_host with the attention of
 * head group fail_group (0 <= fail_group < h3attn_forward_host_groups(H, heads_per_group,
 * NULL)) launched through
 * h3attn_debug_attend_timeout (waits bounded by wait_limit_ns, 1 ms to 2 s, the O-ready
 * arrivals withheld), every other group as usual.  h3attn_forward_host_check_status then
 * reports H3ATTN_ERR_TIMEOUT, whichever group failed; the other groups' output heads are
 * those of h3attn_forward_host.  No fault, trap or unbounded wait is involved. */
h3attn_status h3attn_debug_forward_host_timeout(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                                const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H,
                                                int D, float softmax_scale, const h3attn_bf16_out* out,
                                                int heads_per_group, void* dev_buf, size_t dev_bytes,
                                                int fail_group, uint64_t wait_limit_ns, void* stream);

/* Failure-path test hook: h3attn_attend with every barrier wait bounded by
 * wait_limit_ns (1 ms to 2 s) and the correction warpgroup's "O ready" arrivals
 * withheld, so that the PV issuer's wait, and every wait behind it, has no
 * producer.  The first of them to run out records H3ATTN_ERR_TIMEOUT in the
 * workspace status word (detail word: its wait-site id; block word: its CTA),
 * raises its CTA's abort flag, and every role of the CTA drains the copies and
 * tensor-core work it started, frees the tensor memory and returns; no fault,
 * trap or unbounded wait is involved, and the CUDA context stays usable.
 * Returns H3ATTN_OK when the launch was made; h3attn_check_status then reports
 * H3ATTN_ERR_TIMEOUT.  Output rows are unspecified.  Arguments as h3attn_attend.
 * Tests the failure side of the no-deadlock requirement of "Phase 2B Aligned
 * Numerical Prototype", Exactness: a wait whose producer never arrives ends with
 * an error status instead of a hang. */
h3attn_status h3attn_debug_attend_timeout(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H,
                                          int D, float softmax_scale, const h3attn_bf16_out* out,
                                          uint64_t wait_limit_ns, void* stream);

/* Tracing export: h3attn_attend with a timeline probe in one CTA (linear block index
 * trace_block; CTAs are (pair of 128-row Q tiles, head, batch), pair fastest).  Writes clock64()
 * stamps of 16 events for each key tile j to trace_dev[(event*2 + slot)*ceil(Tkv/128) + j]
 * (uint64, device memory, 32*ceil(Tkv/128) entries; entries of events that did not
 * happen are left untouched).  slot = the Q tile of the pair (0 or 1) the event belongs to;
 * K-tile events use slot 0.  Events: 0 scores ready in the softmax warpgroup, 1 running max
 * of tile j published to the correction, 2 probabilities handed to the PV issuer, 3 QK
 * issued, 4 PV issued, 5 O rescaled (or left alone) by the correction warpgroup, 6 K tile
 * landed, 7 probabilities computed (end of the MUFU turn), 8 PV issued and committed,
 * 9 scores released (QK of tile j+1 may start), 10 scores in registers, 11 own row maxima
 * known, 12 probability buffer free (PV of tile j-1 completed), 13 the PV issuer saw the
 * probabilities, 14 the PV issuer saw O ready, 15 probabilities handed over by the softmax
 * warp of the last row quarter (events 0-2, 7, 10-12 are the first quarter's).
 * Reproduces the QK/PV overlap measurement of "Phase 2B Aligned Numerical Prototype",
 * Synchronization And Safety.  Same output as h3attn_attend. */
h3attn_status h3attn_debug_attend_trace(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H,
                                        int D, float softmax_scale, const h3attn_bf16_out* out,
                                        int trace_block, uint64_t* trace_dev, void* stream);

/* Size of the device array behind h3attn_forward_static (64 MiB). */
#define H3ATTN_STATIC_WS_BYTES (64u << 20)

/* H3ATTN_STATIC_WS_BYTES as compiled into the loaded library. */
size_t h3attn_static_workspace_bytes(void);

/* Forward pass (quantize + attend, Tq and Tkv as in h3attn_forward_ex) for callers that
 * cannot allocate device memory: a host that owns the device allocator and offers this
 * library no way to request memory, or a runtime that forbids allocation after start-up.
 * The pages have no counterpart; it is an interface addition of this library.
 * Takes the inputs and the output only. The workspace is a file-scope device array of
 * H3ATTN_STATIC_WS_BYTES that every GPU loading the library holds until exit; shapes
 * whose h3attn_workspace_bytes exceeds it return H3ATTN_ERR_WORKSPACE before anything is
 * enqueued. Every call looks up the array's device address for the current device and
 * context (cudaGetSymbolAddress, a host-side query); the first call on a device also makes
 * the runtime load the library's device code there, so make that first call before any
 * stream capture. Calls no cudaMalloc or cudaFree. All calls share the array, which keeps
 * the last call's contents, so calls whose GPU work overlaps race on it; the caller must
 * order them. Device-side wait timeouts are recorded in the array's sticky status word:
 * read it with h3attn_static_check_status. */
h3attn_status h3attn_forward_static(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                    const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                    float softmax_scale, const h3attn_bf16_out* out, void* stream);

/* h3attn_check_status on the static array of h3attn_forward_static (current device):
 * synchronises `stream`, returns the first device-side failure of any static call since
 * the last check (H3ATTN_OK or H3ATTN_ERR_TIMEOUT) and clears it.  Like the entry point
 * it serves, it allocates nothing. */
h3attn_status h3attn_static_check_status(void* stream);

/* Failure-path test hook on the static array: h3attn_debug_attend_timeout run on the
 * workspace that the last h3attn_forward_static call of the same sizes filled.  Sizes
 * that do not fit the array return H3ATTN_ERR_WORKSPACE; h3attn_static_check_status then
 * reports H3ATTN_ERR_TIMEOUT. */
h3attn_status h3attn_debug_static_attend_timeout(int B, int Tq, int Tkv, int H, int D, float softmax_scale,
                                                 const h3attn_bf16_out* out, uint64_t wait_limit_ns,
                                                 void* stream);

/* ---- Q/K RMSNorm + RoPE before the attention ("H3 Performance Roadmap", Component 2
 * execution order, item 1: Q/K normalization and RoPE where the attention consumes Q
 * and K; "Norm and RoPE" in the representative block table).  The pages give no
 * formula; the one implemented, per (b, t, h) row of 128 channels x:
 *   ss  = sum of x_c^2 in FP32 (sixteen 8-channel slice sums, each in channel order,
 *         then added pairwise: slice s += slice s+8 for s < 8, then s += s+4 for s < 4,
 *         s += s+2, s += s+1; every product and sum rounded separately);
 *   r   = 1 / sqrt(ss / 128 + eps)   (FP32; sqrt and division correctly rounded);
 *   z_c = bf16(bf16(x_c * r) * gamma_c);
 *   out_2i   = bf16(z_2i * cos_i - z_2i+1 * sin_i),
 *   out_2i+1 = bf16(z_2i+1 * cos_i + z_2i * sin_i)  (FP32, every product and sum rounded,
 *                                                     no fused multiply-add).
 * Positions are the caller's: row t of the cos/sin tables belongs to token t of every
 * batch item and head (a 3-axis video RoPE, or cos 1 / sin 0 for tokens left
 * unrotated, is encoded in the tables). */
typedef struct {
  const float* gamma_q; /* [128] FP32 RMSNorm weight applied to Q (device, 16-byte aligned) */
  const float* gamma_k; /* [128] FP32 weight applied to K */
  const float* cos_q;   /* [Tq, 64] FP32 rotary tables of the query positions (row-major, */
  const float* sin_q;   /*          device, 16-byte aligned) */
  const float* cos_k;   /* [Tkv, 64] FP32 rotary tables of the key positions */
  const float* sin_k;
  float eps;            /* > 0 and finite */
} h3attn_qk_norm_rope;

/* h3attn_quantize_qkv on the normalized and rotated Q and K (V unchanged).  Four
 * launches: the transform of Q written straight into the workspace's Q-word area; the
 * statistics pass, which transforms K in registers (it needs it for the K means) and
 * leaves it in the K-word area; the ordered reduction; the quantize pass, which reads
 * Q and K from the workspace and overwrites them with the words.  The words are bit for
 * bit those of h3attn_norm_rope on Q and K followed by h3attn_quantize_qkv; the raw Q,
 * K and V are read once and no tensor outside the workspace is written.
 * H3ATTN_ERR_INVALID_ARG for a null nr or table, or eps not > 0 and finite;
 * H3ATTN_ERR_ALIGNMENT for a table not 16-byte aligned. */
h3attn_status h3attn_quantize_qkv_norm_rope(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                            const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                            const h3attn_qk_norm_rope* nr, void* ws, size_t ws_bytes,
                                            void* stream);

/* h3attn_quantize_qkv_norm_rope + h3attn_attend. */
h3attn_status h3attn_forward_norm_rope(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                       const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                       float softmax_scale, const h3attn_qk_norm_rope* nr,
                                       const h3attn_bf16_out* out, void* ws, size_t ws_bytes, void* stream);

/* The transform above as a separate pass: x [B, T, H, 128] -> out (same shape, any
 * strides).  gamma [128], cos/sin [T, 64]: FP32 device arrays, 16-byte aligned.  out
 * may be x itself (in place); partially overlapping views are undefined. */
h3attn_status h3attn_norm_rope(const h3attn_bf16_view* x, int B, int T, int H, int D, const float* gamma,
                               const float* cos_tab, const float* sin_tab, float eps,
                               const h3attn_bf16_out* out, void* stream);

/* Static description of a status code. */
const char* h3attn_status_string(h3attn_status s);

/* H3ATTN_VERSION of the loaded library. */
int h3attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* H3ATTN_H_ */
