/*
 * hv_attn.h - C ABI of the joint 3D-RoPE full-attention library (libhvattn.so).
 *
 * What it computes. For every batch sample b and head h, over the joint
 * sequence [video tokens ; text tokens] (HunyuanVideo 模型结构与数学原理,
 * §5.2 "双流块": Q=[Q_v;Q_t], K=[K_v;K_t], V=[V_v;V_t],
 * Attn = softmax(QK^T/sqrt(128))V, joint length S = N + L):
 *
 *   q'_i = R(t_i,h_i,w_i) q_i for video rows i < N, q'_i = q_i for text rows;
 *   k'_j likewise;                                     (§5.5 "3D RoPE")
 *   out_i = sum_{j < N+valid_b} softmax_j(scale * q'_i . k'_j) v_j.
 *
 * R = R_t (+) R_h (+) R_w acts on the head dimension 128 split into
 * (d_t, d_h, d_w) = (16, 56, 56) channel segments (§5.5; the tech-report
 * summary's Table 2); inside a segment of width d, the adjacent channel pair
 * (2i, 2i+1) turns by pos * theta^(-2i/d) as
 * (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos), pos being the token's
 * t, h or w coordinate. Video tokens are the T x Hp x Wp patch grid flattened
 * t-major, then h, then w (token n: t = n/(Hp*Wp), h = (n/Wp)%Hp, w = n%Wp);
 * text tokens are not rotated. Keys at or past N + text_valid[b] (text
 * padding) are masked out; every query row, padded text rows included, is
 * computed and written.
 *
 * All calls are plain C, return an hv_status code, never throw and never
 * abort the process.
 */
#ifndef HV_ATTN_H
#define HV_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum hv_status {
    HV_OK = 0,
    HV_ERR_NULL_POINTER = 1,   /* a required pointer is NULL                        */
    HV_ERR_MISALIGNED = 2,     /* q/k/v/out not 16-byte aligned                      */
    HV_ERR_BAD_SHAPE = 3,      /* B, heads, T, Hp or Wp < 1, or B > HV_MAX_BATCH     */
    HV_ERR_BAD_TEXT = 4,       /* text_len not in [0,256] or text_valid[b] not in [0,text_len] */
    HV_ERR_TOO_LARGE = 5,      /* S*heads*128 or a TMA coordinate exceeds int32      */
    HV_ERR_ALIAS = 6,          /* out overlaps q, k, v (or qk_gamma)                 */
    HV_ERR_BAD_SCALAR = 7,     /* rope_theta <= 0 or not finite, scale not finite, qk_eps < 0 or not finite */
    HV_ERR_NO_DEVICE = 8,      /* current CUDA device is not an sm_100 (B200) part   */
    HV_ERR_LAUNCH = 9,         /* a CUDA runtime/driver call failed                  */
    HV_ERR_DEVICE_TIMEOUT = 10,/* a kernel-side wait ran out (see hv_attn_last_device_error) */
    HV_ERR_WORKSPACE = 11,     /* workspace NULL, not 16-byte aligned, too small or overlapping */
    HV_ERR_NOALLOC_LIMIT = 12  /* problem too large for hv_attn_forward_noalloc's built-in scratch */
};

#define HV_HEAD_DIM 128
#define HV_MAX_TEXT_LEN 256
#define HV_MAX_BATCH 512

/*
 * hv_attn_forward - joint full self-attention with 3D RoPE on the video rows.
 *
 * q, k, v  : device pointers, bf16, layout [B, S, heads, 128] row-major and
 *            contiguous (S = T*Hp*Wp + text_len; the last three dims
 *            [S, heads, 128] as in §5.6 "用张量形状读一个 Transformer block"),
 *            video tokens first, then text_len text tokens (valid first,
 *            padding last). Un-rotated: the call applies the rotation.
 *            Padded text rows of k and v must hold finite values (they get
 *            probability 0, and 0 * NaN would still poison the sum).
 * out      : device pointer, bf16, same layout; every row is written.
 *            Must not overlap q, k or v.
 * B, heads : batch and head count (>= 1, B <= HV_MAX_BATCH).
 * T, Hp, Wp: video-token grid (T' = floor((F-1)/4)+1, Hp = H/16, Wp = W/16
 *            for an F x H x W clip; see hv_video_tokens), each >= 1.
 * text_len : text tokens per sample in the buffers, 0..256 (the MLLM branch
 *            keeps at most 256 prompt tokens, §3.1).
 * text_valid: HOST pointer to B ints, 0 <= text_valid[b] <= text_len; read
 *            before the call returns (the caller may free it right after).
 * rope_theta: RoPE base (> 0; the pages' default is 256).
 * scale    : softmax scale (finite; the pages use 1/sqrt(128)).
 * cuda_stream: cudaStream_t to enqueue on (NULL = legacy default stream).
 *
 * Ownership: the caller owns all buffers; the library allocates no device
 * memory. Asynchronous: enqueues one kernel and returns without
 * synchronising. Errors in the arguments are reported before anything is
 * launched. A kernel-side wait that runs out (a broken pipeline, never an
 * expected event) sets the device error word read by
 * hv_attn_last_device_error and a status word in host memory; the kernel then
 * ends cleanly. While that status word is set, every entry point that
 * launches work on the device returns HV_ERR_DEVICE_TIMEOUT without
 * launching (checked without synchronising), until hv_attn_last_device_error
 * reads and clears it. The status words live in one static 4 KB page of host
 * memory that the first call on a device page-locks and maps for the device
 * (cudaHostRegister: a registration, not an allocation); make that first call
 * before any stream capture.
 */
int hv_attn_forward(const void* q, const void* k, const void* v, void* out,
                    int B, int heads, int T, int Hp, int Wp,
                    int text_len, const int* text_valid,
                    float rope_theta, float scale, void* cuda_stream);

/*
 * hv_attn_forward_ws - the same result as hv_attn_forward, in two stages:
 * a memory-bound kernel first writes the rotated keys R(K) (video rows
 * rotated exactly as hv_attn_forward rotates them, text rows copied) into
 * `workspace`, then the attention kernel reads them and rotates only Q as it
 * loads it. The output is bit-identical to hv_attn_forward's. This trades
 * workspace_bytes >= hv_attn_workspace_bytes(...) of device memory and one
 * extra read and write of K (HBM traffic of 2 * B*S*heads*256 bytes) for
 * taking the per-tile key rotation out of the attention loop (§5.5 "3D
 * RoPE" applies R to K once; it does not say where).
 *
 * workspace: device pointer owned by the caller, 16-byte aligned, not
 *            overlapping q, k, v or out; its contents on return are R(K).
 * Other arguments, ownership, asynchrony and errors as hv_attn_forward;
 * HV_ERR_WORKSPACE for a bad workspace. Two kernels are enqueued on the
 * stream, in order.
 */
int hv_attn_forward_ws(const void* q, const void* k, const void* v, void* out,
                       int B, int heads, int T, int Hp, int Wp,
                       int text_len, const int* text_valid,
                       float rope_theta, float scale,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * hv_attn_forward_qknorm - hv_attn_forward with the per-head QK RMSNorm
 * prologue of the DiT blocks (§5.4 "归一化、条件调制和残差门": RMSNorm on the Q
 * and K of every attention head): before the rotation, every Q and K row
 * (one token, one head, 128 channels) becomes
 *   y = gamma * x / sqrt((1/128) sum_j x_j^2 + eps),
 * video rows with the video stream's gamma and text rows with the text
 * stream's (the double-stream blocks keep separate parameters per modality,
 * §5.2; a single-stream block passes the same gamma twice). Then video rows
 * are rotated as in hv_attn_forward and attention is computed on the result.
 * The normalised, rotated rows are rounded to bf16 once, as the rotation
 * alone is.
 *
 * qk_gamma : DEVICE pointer, fp32 [4][128], 16-byte aligned, owned by the
 *            caller: gamma of Q video rows, K video rows, Q text rows, K text
 *            rows, in that order; shared by all heads. Must not overlap out.
 * qk_eps   : epsilon inside the root (finite, >= 0; the pages give no value,
 *            1e-6 is usual).
 * Other arguments, asynchrony and errors as hv_attn_forward;
 * HV_ERR_NULL_POINTER / HV_ERR_MISALIGNED / HV_ERR_BAD_SCALAR / HV_ERR_ALIAS
 * also cover qk_gamma and qk_eps.
 *
 * Two kernels: the first computes every key row's factor 1/rms once (reads
 * K once), the attention kernel scales each K tile by them as it lands,
 * instead of reducing every key row again for every 256-row query unit.
 * Ownership: the caller owns all buffers. The row factors take
 * 4 * B * heads * ceil(S/128) * 128 bytes of stream-ordered scratch
 * (cudaMallocAsync on cuda_stream from the device's default memory pool,
 * cudaFreeAsync on the same stream right after the attention kernel is
 * enqueued); if the pool cannot provide it the call returns HV_ERR_LAUNCH
 * before launching anything. Callers that must not allocate use
 * hv_attn_forward_qknorm_ws with a workspace of their own.
 */
int hv_attn_forward_qknorm(const void* q, const void* k, const void* v, void* out,
                           int B, int heads, int T, int Hp, int Wp,
                           int text_len, const int* text_valid,
                           float rope_theta, float scale,
                           const float* qk_gamma, float qk_eps, void* cuda_stream);

/*
 * hv_attn_forward_qknorm_ws - hv_attn_forward_qknorm in the two stages of
 * hv_attn_forward_ws: the first kernel writes the normalised, rotated keys
 * into `workspace` (text rows normalised), the attention kernel normalises
 * and rotates Q on load. Output bit-identical to hv_attn_forward_qknorm.
 * Arguments as hv_attn_forward_qknorm plus workspace / workspace_bytes as in
 * hv_attn_forward_ws (the workspace must not overlap qk_gamma either). It
 * allocates no device memory.
 */
int hv_attn_forward_qknorm_ws(const void* q, const void* k, const void* v, void* out,
                              int B, int heads, int T, int Hp, int Wp,
                              int text_len, const int* text_valid,
                              float rope_theta, float scale,
                              const float* qk_gamma, float qk_eps,
                              void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * hv_attn_workspace_bytes - workspace hv_attn_forward_ws needs:
 * B * (T*Hp*Wp + text_len) * heads * 128 * 2 bytes; -1 for a bad shape.
 */
long long hv_attn_workspace_bytes(int B, int heads, int T, int Hp, int Wp, int text_len);

/*
 * hv_attn_forward_noalloc - hv_attn_forward_ws with no workspace argument and
 * no allocation: the rotated keys go to a scratch array built into the
 * library (HV_NOALLOC_MAX_BYTES = 64 MiB of device memory per device that
 * loads the library, held until the process exits).
 *
 * No counterpart in the paper: this entry point exists for callers that
 * cannot allocate device memory when they call attention - for example an
 * application whose own allocator owns the device memory and forbids other
 * allocations, or a tight loop that must not pay for cudaMalloc's implicit
 * synchronisation - and that have no spare buffer to hand in as workspace.
 *
 * Arguments, result (bit-identical to hv_attn_forward) and errors as
 * hv_attn_forward. Problems needing more than HV_NOALLOC_MAX_BYTES of
 * rotated keys (B * S * heads * 256 bytes) are rejected with
 * HV_ERR_NOALLOC_LIMIT before anything is launched. It calls no cudaMalloc,
 * cudaFree or other allocating routine. Every call looks up the scratch
 * array's device address in the current context (cudaGetSymbolAddress); the
 * first call on a device also loads the library's kernels there, so make it
 * before any stream capture. Every call on a
 * device shares the one scratch array, which keeps the last call's contents:
 * calls whose kernels overlap on the GPU (different streams, or different
 * host threads) race on it and must be ordered by the caller.
 */
#define HV_NOALLOC_MAX_BYTES (64ull << 20)
int hv_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out,
                            int B, int heads, int T, int Hp, int Wp,
                            int text_len, const int* text_valid,
                            float rope_theta, float scale, void* cuda_stream);

/*
 * hv_attn_forward_host - the whole call from and to HOST memory, with the
 * copies overlapping the attention kernel. The heads are cut into
 * `head_groups` groups (heads % head_groups == 0), and the first and the
 * last group further into one head and the rest, so that only one head's
 * columns are copied in before the first kernel and out after the last.
 * Per piece, in a pipeline of two device staging slots: a 2-D copy of the
 * piece's q, k, v columns host -> device, the attention kernel on the
 * contiguous [B, S, heads_of_piece, 128] staging tensors, and a 2-D copy of
 * its output columns back into out_host. The kernels of consecutive pieces
 * alternate between two streams, so that one piece's kernel takes the SMs
 * the previous one frees during its last wave. Heads are independent (§5.2
 * computes attention per head), so the result equals hv_attn_forward's bit
 * for bit. No counterpart in the pages: it is the host-buffer form of the
 * same call.
 *
 * q_host, k_host, v_host, out_host: HOST pointers, layout as hv_attn_forward;
 *            page-locked (pinned) memory lets the copies run asynchronously;
 *            out_host must not overlap the inputs.
 * head_groups: >= 1, dividing heads.
 * workspace: DEVICE pointer, 16-byte aligned, at least
 *            hv_attn_host_workspace_bytes(...) bytes, owned by the caller.
 * cuda_stream: the copies and kernels run on four streams the library
 *            creates once per device (copies in, copies out, two for the
 *            kernels; make the first call before any stream capture), ordered
 *            after the work already enqueued on `cuda_stream`. The call is
 *            asynchronous: `cuda_stream` is made to wait for the last copy, so
 *            out_host is complete once that stream has been synchronised; the
 *            host buffers must stay valid until then. Calls on one device
 *            share these streams and are enqueued one at a time (a mutex), so
 *            they run in turn.
 * Errors: HV_ERR_NULL_POINTER, HV_ERR_BAD_SHAPE (also bad head_groups),
 * HV_ERR_BAD_TEXT, HV_ERR_ALIAS (host buffers), HV_ERR_WORKSPACE, and those of
 * hv_attn_forward for one group's call; HV_ERR_LAUNCH if a copy or a stream
 * operation fails.
 */
int hv_attn_forward_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                         int B, int heads, int T, int Hp, int Wp,
                         int text_len, const int* text_valid,
                         float rope_theta, float scale, int head_groups,
                         void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * hv_attn_host_workspace_bytes - device workspace hv_attn_forward_host needs:
 * 8 * B * S * (heads / head_groups) * 128 * 2 bytes (two slots of q, k, v, out);
 * -1 for a bad shape or head_groups.
 */
long long hv_attn_host_workspace_bytes(int B, int heads, int T, int Hp, int Wp, int text_len, int head_groups);

/*
 * hv_attn_forward_block - one step of ring attention (§9.2 "xDiT/USP 序列并行":
 * each rank keeps a run of query rows while K/V blocks pass around the ring):
 * attention of a block of Sq query rows against a block of Sk key/value rows,
 * plus the log-sum-exp of every query row, so that the results of several
 * key blocks can be merged (hv_attn_merge).
 *
 * Both blocks are runs of consecutive rows of the joint sequence of the
 * T x Hp x Wp grid: the first q_video (k_video) rows are video tokens whose
 * global token indices are q_pos0, q_pos0 + 1, ... (k_pos0, ...), rotated by
 * the 3D RoPE of those tokens; the remaining rows are text (not rotated).
 * Only the first kv_len[b] key rows of sample b take part.
 *
 * q        : device bf16 [B, Sq, heads, 128]; k, v: device bf16 [B, Sk, heads, 128].
 * out      : device [B, Sq, heads, 128], bf16 (out_fp32 = 0) or fp32 (out_fp32 = 1:
 *            the block's partial result kept at full precision for hv_attn_merge,
 *            so that a long ring adds no bf16 rounding per step).
 * lse      : device fp32 [B, Sq, heads] or NULL; lse = log(sum_j exp(s_j)) of
 *            the scaled scores s_j = scale * q'.k'_j over the block's keys.
 * kv_len   : HOST pointer to B ints, 1 <= kv_len[b] <= Sk (a block with no
 *            key at all has no result; leave it out of the merge).
 * Constraints: 0 <= q_video <= Sq, 0 <= k_video <= Sk, q_pos0, k_pos0 >= 0 and
 * q_pos0 + q_video, k_pos0 + k_video <= T*Hp*Wp (HV_ERR_BAD_SHAPE otherwise);
 * kv_len out of range: HV_ERR_BAD_TEXT; out or lse overlapping an input or
 * each other: HV_ERR_ALIAS. Other errors, ownership and asynchrony as
 * hv_attn_forward. hv_attn_forward is the special case Sq = Sk = S,
 * q_video = k_video = N, offsets 0, kv_len[b] = N + text_valid[b].
 */
int hv_attn_forward_block(const void* q, const void* k, const void* v, void* out, float* lse,
                          int B, int heads, int T, int Hp, int Wp,
                          int Sq, int q_video, int q_pos0, int Sk, int k_video, int k_pos0,
                          const int* kv_len, float rope_theta, float scale, int out_fp32,
                          void* cuda_stream);

/*
 * hv_attn_merge - fold one key block's result (o_part, fp32 if o_part_fp32 = 1
 * else bf16; lse_part fp32) into the running result (o_acc fp32, lse_acc fp32)
 * of the same `rows` query rows of 128 channels: with m = max(lse_acc,
 * lse_part), w = exp(lse - m),
 *   o_acc <- (w_acc o_acc + w_part o_part) / (w_acc + w_part),
 *   lse_acc <- m + log(w_acc + w_part),
 * the softmax over the union of the keys. Start from o_acc = 0 and
 * lse_acc = -inf. If `out` is not NULL the merged rows are also written to it
 * as bf16 (the last merge of a ring). Device pointers; o_acc 16-byte, o_part
 * 16-byte (fp32) or 8-byte (bf16), out 8-byte, lse 4-byte aligned.
 * Asynchronous on cuda_stream. No counterpart in the pages beyond the merge
 * rule of ring attention.
 */
int hv_attn_merge(float* o_acc, float* lse_acc, const void* o_part, int o_part_fp32, const float* lse_part,
                  void* out, long long rows, void* cuda_stream);

/*
 * hv_video_tokens - number of video tokens N = (floor((F-1)/4)+1)*(H/16)*(W/16)
 * of an F x H x W clip (§4 "Causal 3D VAE": temporal compression 4 keeping the
 * first frame, spatial 8, then the 1x2x2 patch). Returns -1 when F is not
 * 4k+1 (k >= 0) or H, W are not positive multiples of 16. Pure host function.
 */
long long hv_video_tokens(int frames, int height, int width);

/*
 * hv_attn_last_device_error - synchronises the current device, returns the
 * device-side error word accumulated by kernels of this library since the
 * previous call, and clears it together with the device's host status word
 * (after which the entry points launch again). 0 = none. Otherwise bit 0 is
 * set for a wait that ran out, and bits 8..15 name the waiting role
 * (1 producer, 2 MMA, 3 softmax, 4 RoPE, 5 self-test; several roles OR
 * together). Returns -1 if the device cannot be read.
 */
int hv_attn_last_device_error(void);

/*
 * hv_attn_selftest_timeout - launches a one-warp kernel whose bounded wait on
 * an mbarrier that nothing completes must run out after about timeout_us
 * microseconds, then synchronises and returns the device error word that run
 * left (expected: bit 0 set, role 5). Tests the timeout path without faulting
 * or hanging the GPU. Returns -1 on a CUDA error.
 */
int hv_attn_selftest_timeout(int timeout_us);

/*
 * hv_attn_selftest_abort - a test of the attention kernel's own abort path,
 * without faulting or hanging anything: runs hv_attn_forward's kernel (keys
 * rotated on load, rope_theta 256, scale 1/sqrt(128)) on the caller's problem
 * with every wait bounded by timeout_us microseconds (1000..1000000) and with
 * CTA 0 leaving its K tile load number withhold_k (>= 0, counted over that
 * CTA's loads) unissued, so that a wait runs out: the RoPE warps' for those
 * keys, or the producer's for the stage they hold (whichever polls first
 * past the limit records its role). That CTA then stops every role, lets
 * its copies and MMAs in
 * flight finish, frees its TMEM and returns, while the other CTAs finish. Synchronises `cuda_stream`, then returns HV_OK;
 * the error word and the host status word are set as for any timeout (read
 * and clear them with hv_attn_last_device_error). `out` is left partly
 * written. Arguments as hv_attn_forward; HV_ERR_BAD_SCALAR for a bad
 * withhold_k or timeout_us.
 */
int hv_attn_selftest_abort(const void* q, const void* k, const void* v, void* out,
                           int B, int heads, int T, int Hp, int Wp,
                           int text_len, const int* text_valid, int withhold_k, int timeout_us,
                           void* cuda_stream);

/* Static string for an hv_status code. */
const char* hv_attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* HV_ATTN_H */
