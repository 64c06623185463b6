/*
 * vdn.h - C ABI of libvdn: the Video DeltaNet hybrid video-video attention
 * forward on NVIDIA B200 (sm_100a).
 *
 * The operation (sources: the project page "Video DeltaNet: Near-Lossless
 * Hybrid Attention for Video Models", sections "Local Softmax and Long-Range
 * Linear Memory", "Gating the Softmax and Linear Branch Outputs" and "Video
 * Delta Attention: A Frame-Wise Solution"; and "Faster Than It Plays", section
 * "Two branches instead of one", for the closed form S = (S_bar + B)(I + A)^-1):
 *
 *   softmax branch  o_soft = softmax(q K^T / sqrt(d)) V over the key set of the
 *                   query's frame: the frames of its chunk and of the two
 *                   neighbouring chunks, the boundary frames 0 and F-1, and all
 *                   T text tokens (one normaliser). Boundary-frame queries see
 *                   every frame.
 *   linear branch   Video Delta Attention: per frame, A = K^T Diag(beta) K,
 *                   B = V^T Diag(beta) K, S <- (S + B)(I + A)^-1; a forward scan
 *                   over frames 1, 2, ... and a reverse scan over F-2, F-3, ...,
 *                   both starting from S0 = 1/2 B_T (I + A_T)^-1 (the text
 *                   written once into a zero state, halved). A non-boundary
 *                   frame whose window is frames [lo, hi] reads the forward
 *                   state after frames 1..lo-1 and the reverse state after
 *                   frames F-2..hi+1 (S0 where empty): o_lin = (S_fwd + S_rev) q.
 *                   Boundary frames (0 and F-1) are never scanned and have
 *                   o_lin = 0.
 *   combine         out = sigmoid(g_s) * o_soft + sigmoid(g_l) * RMSNorm_d(o_lin)
 *                   (element-wise gates; RMSNorm over the head dim with eps and
 *                   an optional weight).
 *
 * Layout. Chunk of frame f: ch(f) = f / c (integer division; the last chunk is
 * partial when c does not divide F). L = F * N video tokens, token index
 * f * N + n (frame-major). All tensors are dense, row-major:
 *   q, k, v, g_soft, g_lin, out, out_soft, out_lin, o_soft, o_lin : [B, L, H, d]
 *   k_text, v_text                                                 : [B, T, H, d]
 *   beta  : [B, L, H] float32      beta_text : [B, T, H] float32
 *   lse   : [B, L, H] float32 (natural-log normaliser of the softmax branch)
 *   chunk_states : [B, H, 2, J, d, d] float32, J = ceil(F / c); [.., 0, j] is the
 *                  forward and [.., 1, j] the reverse state read by chunk j
 *                  (row index = value dim, column = key dim). Entries of chunks
 *                  that hold no non-boundary frame are zero.
 * Tensors of element type vdn_dtype_t are float32 (VDN_F32) or bfloat16
 * (VDN_BF16); accumulation, softmax statistics and VDA states are float32.
 * Inputs are used as given: the library does not normalise k or rescale q.
 *
 * Supported: VDN_F32 with d in {16, 32, 64, 128}; VDN_BF16 with d in {64, 128}.
 * T may be 0 (k_text, v_text, beta_text may then be NULL).
 *
 * Ownership and execution. Every pointer is caller-owned device memory, except
 * the layout struct which is read on the host during the call. The library
 * allocates no memory and keeps no state between calls besides a device-side
 * status word (vdn_device_status) and the static scratch array used by
 * vdn_vda_scan_fwd_noalloc (and the host-buffer entry's streams, below).
 * Calls are asynchronous on `stream`;
 * the return code reports host-detectable errors (VDN_ERR_INVALID for a bad
 * layout or a NULL required pointer, VDN_ERR_UNSUPPORTED for a dtype/d
 * combination not built or a pointer not 16-byte aligned, VDN_ERR_WORKSPACE
 * for a short workspace) and launch errors (VDN_ERR_CUDA). On any error
 * nothing is launched, except for VDN_ERR_CUDA where kernels launched before
 * the failing one may run.
 */
#ifndef VDN_H_
#define VDN_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int B;  /* batch */
  int F;  /* latent frames */
  int N;  /* video tokens per frame */
  int T;  /* text tokens */
  int c;  /* frames per chunk */
  int H;  /* heads */
  int d;  /* head dim (shared by q, k, v) */
} vdn_layout_t;

typedef enum { VDN_F32 = 0, VDN_BF16 = 1 } vdn_dtype_t;

typedef enum {
  VDN_OK = 0,
  VDN_ERR_INVALID = 1,
  VDN_ERR_UNSUPPORTED = 2,
  VDN_ERR_WORKSPACE = 3,
  VDN_ERR_CUDA = 4,
  VDN_ERR_TIMEOUT = 5,
  VDN_ERR_BOUNDS = 6   /* only from a library built with bound checks (see below) */
} vdn_status_t;

/* Bytes of device workspace that vdn_vda_scan_fwd and vdn_hybrid_attn_fwd (and
 * their _decay forms) need for this layout and dtype (the maximum of the two).
 * 0 for an invalid layout. */
size_t vdn_workspace_bytes(const vdn_layout_t* layout, int dtype);

/* Softmax branch alone (project page, "Local Softmax and Long-Range Linear
 * Memory"): o_soft = softmax over the window + anchor frames + text keys,
 * ungated. lse (nullable) receives the natural-log normaliser per query. */
int vdn_window_softmax_fwd(const vdn_layout_t* layout, int dtype,
                           const void* q, const void* k, const void* v,
                           const void* k_text, const void* v_text,
                           void* o_soft, float* lse, cudaStream_t stream);

/* Linear branch alone (project page, "Video Delta Attention: A Frame-Wise
 * Solution"; "Faster Than It Plays", closed form): frame Gram matrices, the
 * two scans from the half-weight text state, and the readout o_lin =
 * (S_fwd + S_rev) q, ungated and before RMSNorm (0 for boundary frames).
 * chunk_states (nullable) receives the per-chunk read states. */
int vdn_vda_scan_fwd(const vdn_layout_t* layout, int dtype,
                     const void* q, const void* k, const void* v,
                     const void* k_text, const void* v_text,
                     const float* beta, const float* beta_text,
                     void* o_lin, float* chunk_states,
                     void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The whole hybrid forward (project page, sections "Local Softmax ..." and
 * "Gating the Softmax and Linear Branch Outputs"): out = sigmoid(g_soft) *
 * o_soft + sigmoid(g_lin) * RMSNorm(o_lin). rms_weight (nullable, [d] float32)
 * defaults to ones. out_soft and out_lin (nullable) receive the two gated
 * branches separately (out = out_soft + out_lin), for callers that apply a
 * separate output projection per branch. */
int vdn_hybrid_attn_fwd(const vdn_layout_t* layout, int dtype,
                        const void* q, const void* k, const void* v,
                        const void* k_text, const void* v_text,
                        const float* beta, const float* beta_text,
                        const void* g_soft, const void* g_lin,
                        const float* rms_weight, float rms_eps,
                        void* out, void* out_soft, void* out_lin,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The hybrid forward on tensors in HOST memory (same arguments and layouts as
 * vdn_hybrid_attn_fwd, every tensor pointer a host pointer; rms_weight, if
 * given, a host array of d floats). The call copies in, computes and copies
 * the output back, in chunks of head_chunk heads (<= 0: about ten chunks)
 * pipelined on three internal streams so that the copies of one chunk overlap
 * the kernels of the next (a chunk's k, v and beta are copied first, then q,
 * then the gates, and its kernels start as their own inputs arrive); the heads
 * are independent, so the result equals
 * vdn_hybrid_attn_fwd's bit for bit. Host memory should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to overlap. workspace:
 * device memory of vdn_hybrid_host_workspace_bytes bytes (two chunk buffers).
 * Synchronous: returns when out holds the result. The three streams and their
 * events are created by the first call on a device and kept until the process
 * exits; calls on one device from several host threads take turns. Errors as
 * vdn_hybrid_attn_fwd (validation before any copy). */
size_t vdn_hybrid_host_workspace_bytes(const vdn_layout_t* layout, int dtype, int head_chunk);
int vdn_hybrid_attn_fwd_host(const vdn_layout_t* layout, int dtype, int head_chunk,
                             const void* q, const void* k, const void* v,
                             const void* k_text, const void* v_text,
                             const float* beta, const float* beta_text,
                             const void* g_soft, const void* g_lin,
                             const float* rms_weight, float rms_eps,
                             void* out, void* workspace, size_t workspace_bytes);

/* Linear branch with KDA channel decay (project page "Video DeltaNet", section
 * "Video Delta Attention: A Frame-Wise Solution": the inherited state is decayed
 * per key channel before a frame is written, S_bar = S Diag(alpha)). Same as
 * vdn_vda_scan_fwd except that every scan step over video frame f computes
 * S <- (S Diag(alpha_f) + B_f)(I + A_f)^-1; the text write that makes S0 is not
 * decayed. alpha: [B, F, H, d] float32, required (VDN_ERR_INVALID if NULL),
 * 16-byte aligned, indexed by the key dim (columns of S); values are used as
 * given (the pages take them in (0, 1]; 1 everywhere gives vdn_vda_scan_fwd's
 * result). Entries of the boundary frames 0 and F-1 are never read. */
int vdn_vda_scan_fwd_decay(const vdn_layout_t* layout, int dtype,
                           const void* q, const void* k, const void* v,
                           const void* k_text, const void* v_text,
                           const float* beta, const float* beta_text,
                           const float* alpha,
                           void* o_lin, float* chunk_states,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The whole hybrid forward with the KDA-decayed linear branch of
 * vdn_vda_scan_fwd_decay (alpha as there); everything else as vdn_hybrid_attn_fwd. */
int vdn_hybrid_attn_fwd_decay(const vdn_layout_t* layout, int dtype,
                              const void* q, const void* k, const void* v,
                              const void* k_text, const void* v_text,
                              const float* beta, const float* beta_text,
                              const float* alpha,
                              const void* g_soft, const void* g_lin,
                              const float* rms_weight, float rms_eps,
                              void* out, void* out_soft, void* out_lin,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Softmax branch with FP8 operands (the FP8 attention of the pages' serving
 * stack, "Faster Than It Plays" and the H3 serving notes): q, k, v, k_text,
 * v_text are float8 e4m3 tensors (1 byte per element, same [B, L, H, d] and
 * [B, T, H, d] layouts) with one scale per tensor: value = e4m3 * scale; the
 * text keys and values share k_scale and v_scale. Same key sets and one
 * normaliser as vdn_window_softmax_fwd; scores and softmax statistics in
 * float32, the softmax weights rounded to e4m3 for the P.V product (the row
 * sum adds them before rounding). o_soft: bf16 [B, L, H, d]; lse (nullable)
 * as in vdn_window_softmax_fwd. d must be 128 (VDN_ERR_UNSUPPORTED otherwise);
 * scales must be finite and positive (VDN_ERR_INVALID). */
int vdn_window_softmax_fwd_fp8(const vdn_layout_t* layout,
                               const void* q, const void* k, const void* v,
                               const void* k_text, const void* v_text,
                               float q_scale, float k_scale, float v_scale,
                               void* o_soft, float* lse, cudaStream_t stream);

/* The other tokens of a joint text-video-audio attention layer (project page
 * "Video DeltaNet", attention-map paragraph of "Local Softmax and Long-Range
 * Linear Memory"; "Video DeltaNet speeds MiniMax H3 video generation 14.5x",
 * key facts: the hybrid replaces only video-to-video attention, interactions
 * involving text or audio keep the original softmax).
 *   Audio keys: every video query's softmax also runs over all A audio tokens
 *     (after the text keys, one normaliser). Audio is never written into the
 *     VDA states; only the text prompt initialises them.
 *   Context query rows: the text query rows (q_text, T rows) and the audio
 *     query rows (q_audio, A rows) get the dense softmax over every key of the
 *     layer (all L video, T text and A audio tokens), scale 1/sqrt(d), no gates
 *     and no linear branch, written to o_text / o_audio in the io dtype, with
 *     the natural-log normaliser in lse_text / lse_audio when given.
 * Tensors are dense and row-major like the video ones: [B, T, H, d] for
 * q_text/o_text, [B, A, H, d] for q_audio/k_audio/v_audio/o_audio, [B, T, H]
 * and [B, A, H] float32 for the lse outputs; 16-byte aligned; caller-owned
 * device memory. A NULL q_text (or T = 0) skips the text rows and a NULL
 * q_audio (or A = 0) the audio rows; o_text / o_audio are then not touched.
 * k_audio and v_audio are required when A > 0. */
typedef struct {
  int A;                  /* audio tokens, 0 <= A <= 2^30 */
  const void* k_audio;    /* [B, A, H, d] */
  const void* v_audio;    /* [B, A, H, d] */
  const void* q_text;     /* nullable [B, T, H, d] */
  const void* q_audio;    /* nullable [B, A, H, d] */
  void* o_text;           /* [B, T, H, d], required with q_text when T > 0 */
  void* o_audio;          /* [B, A, H, d], required with q_audio when A > 0 */
  float* lse_text;        /* nullable [B, T, H] */
  float* lse_audio;       /* nullable [B, A, H] */
} vdn_context_t;

/* Softmax part of a joint layer: vdn_window_softmax_fwd with the audio keys
 * added to every video query's key set, plus the dense context query rows
 * (vdn_context_t). ctx is required (VDN_ERR_INVALID if NULL). One launch: the
 * context rows are extra query groups of the same grid. */
int vdn_joint_softmax_fwd(const vdn_layout_t* layout, int dtype, const vdn_context_t* ctx,
                          const void* q, const void* k, const void* v,
                          const void* k_text, const void* v_text,
                          void* o_soft, float* lse, cudaStream_t stream);

/* The attention of a joint text-video-audio layer: video rows get the hybrid
 * forward of vdn_hybrid_attn_fwd (their softmax branch also sees the audio
 * keys), with the KDA decay of vdn_vda_scan_fwd_decay when alpha is not NULL;
 * text and audio query rows get the dense softmax (vdn_context_t). ctx is
 * required; workspace as for vdn_hybrid_attn_fwd (vdn_workspace_bytes). */
int vdn_joint_attn_fwd(const vdn_layout_t* layout, int dtype, const vdn_context_t* ctx,
                       const void* q, const void* k, const void* v,
                       const void* k_text, const void* v_text,
                       const float* beta, const float* beta_text, const float* alpha,
                       const void* g_soft, const void* g_lin,
                       const float* rms_weight, float rms_eps,
                       void* out, void* out_soft, void* out_lin,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The two branches with a float32 output whatever the input dtype: the same
 * computations as vdn_window_softmax_fwd and vdn_vda_scan_fwd, o_soft / o_lin
 * written as float32 [B, L, H, d] (the form the hybrid entry combines
 * internally). They serve callers that run the branches apart and combine
 * later with vdn_gated_combine_fwd, e.g. the branch-specialised sequence-
 * parallel split (project page, "Parallelization & Few-Step Generation"):
 * rounding each branch to bf16 before the combine would add two roundings of
 * its own to the output, beyond the op's tolerance. Arguments, workspace and
 * errors as the plain entries. */
int vdn_window_softmax_fwd_f32out(const vdn_layout_t* layout, int dtype,
                                  const void* q, const void* k, const void* v,
                                  const void* k_text, const void* v_text,
                                  float* o_soft, float* lse, cudaStream_t stream);
int vdn_vda_scan_fwd_f32out(const vdn_layout_t* layout, int dtype,
                            const void* q, const void* k, const void* v,
                            const void* k_text, const void* v_text,
                            const float* beta, const float* beta_text,
                            float* o_lin, float* chunk_states,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The gated combine alone (project page, "Gating the Softmax and Linear Branch
 * Outputs"): out = sigmoid(g_soft) * o_soft + sigmoid(g_lin) * RMSNorm(o_lin),
 * RMSNorm over the head dim with rms_eps and rms_weight (nullable, [d] float32,
 * defaults to ones). o_soft and o_lin are float32 [tokens, H, d] (the _f32out
 * branch outputs of the same tokens; o_lin zero on boundary frames); g_soft,
 * g_lin and out are [tokens, H, d] in dtype. tokens is any number of (batch,
 * token) rows, e.g. B times the length of a token shard. It finishes the
 * hybrid forward when the two branches were computed apart, for instance on
 * different GPUs of a branch-specialised split, and returned to the token
 * shard that holds the gates. tokens == 0 is a no-op. Errors as
 * vdn_hybrid_attn_fwd. */
int vdn_gated_combine_fwd(long long tokens, int H, int d, int dtype,
                          const float* o_soft, const float* o_lin,
                          const void* g_soft, const void* g_lin,
                          const float* rms_weight, float rms_eps, void* out,
                          cudaStream_t stream);

/* Size of the device scratch array behind vdn_vda_scan_fwd_noalloc: 64 MiB. */
#define VDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* The linear-branch entry point for callers that cannot allocate device
 * memory where they run this op (for example a plugin inside an inference
 * engine that owns all device memory and hands plugins no workspace, or a
 * serving loop that forbids device allocations after start-up because
 * cudaMalloc and cudaFree can synchronise the device). The pages have no
 * counterpart to it; it is an interface variant, not a different computation.
 * Same arguments and results as vdn_vda_scan_fwd without the workspace: the
 * scratch lives in a static device array of VDN_NOALLOC_SCRATCH_BYTES that
 * every GPU loading the library holds until the process exits. It needs
 * 2 B H F d^2 4 bytes, plus B H 2 ceil(F/c) d^2 4 bytes when chunk_states is
 * NULL (each part rounded up to 256); a layout needing more returns
 * VDN_ERR_WORKSPACE and launches nothing. The call allocates nothing. The
 * first call on each device looks up the array's device address; make that
 * first call before any stream capture. All calls share the array and it
 * keeps the last call's contents (nothing in it needs to start at zero):
 * calls that overlap on the GPU race with each other and must be serialised. */
int vdn_vda_scan_fwd_noalloc(const vdn_layout_t* layout, int dtype,
                             const void* q, const void* k, const void* v,
                             const void* k_text, const void* v_text,
                             const float* beta, const float* beta_text,
                             void* o_lin, float* chunk_states, cudaStream_t stream);

/* Reads and clears the device-side status word on the current device
 * (synchronises the device). VDN_ERR_TIMEOUT means a kernel gave up a bounded
 * wait and returned without finishing its tile; the outputs of that call are
 * then undefined. Returns VDN_ERR_CUDA if the status cannot be read. */
int vdn_device_status(void);

/* Static string for a status code. */
const char* vdn_status_string(int status);

/* Limit, in nanoseconds, of the bounded waits between the roles of the
 * tensor-core kernels (producer, MMA issuer, softmax / scaler / drain warps):
 * default 4 s; ns = 0 restores it. Process-wide for the current device; set it
 * only while no call of this library is in flight. It exists to exercise the
 * failure path without a fault: with a limit of a few nanoseconds a kernel
 * gives up its waits, records VDN_ERR_TIMEOUT (vdn_device_status), leaves its
 * tile unfinished and exits cleanly. The waits in which a kernel drains its own
 * copies and MMAs before exit keep the 4 s limit, so no copy lands in shared
 * memory of an exited block and no MMA writes freed TMEM. Returns VDN_OK or
 * VDN_ERR_CUDA. */
int vdn_set_wait_limit_ns(unsigned long long ns);

/* The CUDA runtime's description of the error behind the last VDN_ERR_CUDA
 * returned on the calling host thread (by any entry point), or "no CUDA
 * error". Static string. */
const char* vdn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* VDN_H_ */
