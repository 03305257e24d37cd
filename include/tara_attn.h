/*
 * tara_attn.h -- C ABI of the TARA-biased joint self-attention forward pass.
 *
 * The operation (one joint self-attention layer of a reference-to-video diffusion
 * transformer, forward only):
 *
 *   for every branch b, head h and query token i of the packed joint sequence,
 *     s_ij = dot(Q[b,h,i,:], K[b,h,j,:]) * scale + bias_ij          (j over all N tokens)
 *     O[b,h,i,:]  = sum_j softmax_j(s_ij) * V[b,h,j,:]
 *     LSE[b,h,i]  = ln(sum_j exp(s_ij))
 *
 *   bias_ij = -min(strength * (max(|t_i - t_j| - window, 0) / falloff)^2, cap)
 *               if token i is an output (TARGET) video token and token j belongs to the
 *               selected motion (GUIDE) video
 *               ("TARA: Native Temporal Alignment for MiniMax H3 References",
 *                section "The temporal rule");
 *           = m_i * ln(gain[pic_j])  (+ the same term of every extra chained binding)
 *               if token i is a TARGET token with mask weight m_i and token j belongs to
 *               native Picture pic_j
 *               ("BFS H3 Reference Attention Binding (Experimental)", section "The exact rule");
 *           = 0 for every other edge (text, audio, other videos, target->target, and every
 *               query that is not a TARGET token; same two pages, same sections).
 *
 *   scale defaults to 1/sqrt(head_dim) (the score line of "The temporal rule"); the bias is
 *   added after scaling.  LSE is the natural-log log-sum-exp of the scaled, biased logits,
 *   the quantity the pages' FlashAttention-with-LSE backend merges ("TARA: ...", section
 *   "Three backends").
 *
 * Conventions shared by every entry point:
 *   - Status: 0 on success, a negative TARA_ERR_* code otherwise.  Every argument is checked
 *     before anything is launched; a failed check launches nothing and writes nothing.  No
 *     entry point exits, throws or prints.
 *   - Ownership: the caller owns every buffer.  Device buffers are never freed or retained by
 *     the library beyond the call.  tara_attn_forward keeps one internal per-device workspace
 *     (per metadata set and 128-token tile 4,160 bytes: tile and per-key records, each in
 *     ascending and in descending tile order; with qk_int8,
 *     also 2*B*H*N*D bytes of codes and 4*B*H*(N + N/128) bytes of scales); it is allocated
 *     with cudaMalloc the first time a device sees a given size and reused afterwards, so the
 *     first call on a device (or with a larger size) must not be made while a stream is being
 *     captured.
 *   - Asynchrony: device work is enqueued on `stream` and the call returns without
 *     synchronising.  Calls on different streams of one device share the workspace: each
 *     16-bit call makes its stream wait (an event) for the previous call's kernels before
 *     rewriting it, so such calls run one after the other on the GPU.  Calls made while their
 *     stream is being captured skip that ordering; serialise captured work on one stream.
 */
#ifndef TARA_ATTN_H_
#define TARA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------------- */
#define TARA_OK                   0
#define TARA_ERR_NULL            -1  /* a required pointer is NULL                          */
#define TARA_ERR_SHAPE           -2  /* B/H/N/D inconsistent between tensors, or < 1        */
#define TARA_ERR_DTYPE           -3  /* unknown dtype, or Q/K/V/O dtypes differ             */
#define TARA_ERR_HEAD_DIM        -4  /* D not supported (tensor-core path: 64 or 128)       */
#define TARA_ERR_PARAM           -5  /* window/falloff/strength/cap/gain/scale out of domain */
#define TARA_ERR_ALIGN           -6  /* a device pointer is not 16-byte aligned             */
#define TARA_ERR_SEGMENT         -7  /* packer: bad segment description                     */
#define TARA_ERR_CAPACITY        -8  /* packer: output length does not match the segments   */
#define TARA_ERR_CUDA            -9  /* a CUDA runtime/driver call failed                   */
#define TARA_ERR_DEVICE_TIMEOUT -10  /* a kernel gave up on a bounded wait (see below)      */
#define TARA_ERR_TOO_LARGE      -11  /* a size exceeds what an index type or buffer holds   */
#define TARA_ERR_MASK_LENGTH    -12  /* mask neither one frame nor the 17n+5 shot length    */
#define TARA_ERR_DEBUG_CHECK    -13  /* debug build: a device-side check failed (see below)  */

/* ---- token roles ---------------------------------------------------------------------- */
/* Roles of the tokens of the packed joint sequence ("TARA: ...", opening paragraphs and
 * "The temporal rule"; "BFS H3 Reference Attention Binding", "The exact rule").  Values
 * above TARA_SEG_OTHER_VIDEO are treated as plain tokens (no bias) by the kernels.        */
typedef enum {
  TARA_SEG_TEXT        = 0,
  TARA_SEG_PICTURE     = 1,  /* native Picture reference; pic = 1..9                       */
  TARA_SEG_TARGET      = 2,  /* output (generated) video token                             */
  TARA_SEG_GUIDE       = 3,  /* token of the selected motion <Video N> reference           */
  TARA_SEG_AUDIO       = 4,  /* reference / guide audio, packed natively, never biased     */
  TARA_SEG_OTHER_VIDEO = 5   /* native video reference that is not the motion source       */
} tara_seg;

typedef enum { TARA_BF16 = 0, TARA_FP16 = 1, TARA_FP32 = 2 } tara_dtype;

/* A dense tensor [B][H][N][D], row-major and contiguous, in device memory (host memory for
 * tara_attn_forward_host). */
typedef struct {
  void*      ptr;
  tara_dtype dtype;
  int32_t    B, H, N, D;
} tara_tensor;

/* Per-token metadata of the packed sequence, four device arrays of length N each
 * (structure of arrays; host arrays for tara_attn_forward_host).  batch_stride = 0: one set shared by all B branches (the CFG
 * branches of one shot share their packing); otherwise set b starts at element
 * b * batch_stride of every array and there are B sets.
 *   seg    : tara_seg value per token
 *   time_s : seconds on the shared 24 fps clock after temporal RoPE alignment (only read for
 *            TARGET and GUIDE tokens)
 *   pic    : Picture index 1..9 for PICTURE tokens (0 elsewhere; indices outside 1..9 are
 *            neutral)
 *   m      : mask weight of TARGET tokens, normally in [0,1] (a value outside is used as is) */
typedef struct {
  const uint8_t* seg;
  const float*   time_s;
  const uint8_t* pic;
  const float*   m;
  int32_t        N;
  int64_t        batch_stride;
  /* Masks of the extra (chained) bindings, see tara_params.n_extra_bindings: binding k's
   * weight of token i (set b) is extra_m[k * extra_m_stride + b * batch_stride + i].  Device
   * pointer; may be NULL when there are no extra bindings.                                */
  const float*   extra_m;
  int64_t        extra_m_stride;
} tara_token_meta;

/* Rule parameters.  Defaults ("TARA: ...", "The temporal rule"): window 0.20 s,
 * falloff 0.25 s, strength 2.0, cap 6.0.  gain[i-1] is the gain of Picture i
 * ("BFS H3 Reference Attention Binding", "Inputs you'll set": reference_strength for the
 * chosen Picture, other_reference_strength for the others, 1 = neutral).
 * Domain: falloff > 0; window, strength, cap >= 0; gain > 0; all finite.
 * softmax_scale: 0 selects 1/sqrt(D); otherwise a finite positive value used as is.        */
#define TARA_MAX_EXTRA_BINDINGS 3

typedef struct {
  float window, falloff, strength, cap;
  float gain[9];
  float softmax_scale;
  /* Chained bindings ("BFS H3 Reference Attention Binding", "Common issues": two subjects are
   * two chained binding nodes, and overlapping masks combine their log gains).  gain[] with
   * token_meta.m is the first binding; extra binding k (k < n_extra_bindings <= 3) has its own
   * gains extra_gain[k][i-1] and its own mask (token_meta.extra_m).  A target query i and a
   * key of Picture p then get m_i ln(gain[p-1]) + sum_k m_k,i ln(extra_gain[k][p-1]).        */
  int32_t n_extra_bindings;
  float extra_gain[TARA_MAX_EXTRA_BINDINGS][9];
  /* INT8 QK^T ("TARA: ...", "Three backends": the one-pass kernels run the rule on dense INT8
   * attention).  0: Q K^T in the inputs' 16-bit type.  1: the library quantises Q per token
   * and K per 128-token block to symmetric 8-bit codes (tara_quantize_qk_int8) and runs Q K^T
   * on 8-bit tensor cores; the rule, the softmax and P V are unchanged (P and V 16-bit).
   * bf16/fp16 with D = 128 only; other values, dtypes or head sizes return TARA_ERR_PARAM,
   * TARA_ERR_DTYPE, TARA_ERR_HEAD_DIM.                                                     */
  int32_t qk_int8;
} tara_params;

/* Fill *p with the defaults above (all gains 1, softmax_scale 0, no extra bindings, 16-bit
 * QK^T).  NULL is ignored. */
void tara_default_params(tara_params* p);

/* Human-readable name of a status code (static storage, never NULL). */
const char* tara_status_string(int status);

/* ---- the forward pass ------------------------------------------------------------------ */
/* Computes O and LSE as defined at the top of this file.
 *   Q, K, V : device tensors [B][H][N][D], same shape and dtype.  bf16/fp16 run on the
 *             tensor-core kernels (D = 128: a persistent kernel on SM pairs, one cluster of
 *             two CTAs per two SMs walking (branch, head, four-query-tile) work items; D = 64
 *             and 8-bit Q K^T: one CTA per two query tiles); fp32 runs on the exact CUDA-core
 *             kernel (any D from 1 to 256).  Base pointers 16-byte aligned.
 *   meta    : per-token metadata (device pointers), meta->N == N.
 *   p       : rule parameters (host pointer, read during the call only).
 *   O       : device tensor [B][H][N][D] of the same dtype (written).
 *   LSE     : device float array [B][H][N] (written).
 *   stream  : CUDA stream (cudaStream_t), 0 for the legacy default stream.
 * Every O row and LSE entry is written; no other memory of the caller is touched.
 * Extra bindings: 0..3; their gains follow the same domain; extra_m must be non-NULL and
 * 4-byte aligned when there are any, and extra_m_stride at least the length of one m array.
 * Errors: TARA_ERR_NULL, _SHAPE, _DTYPE, _HEAD_DIM, _PARAM, _ALIGN, _TOO_LARGE (B or H
 * above 65535, B*H or the work items B*H*ceil(ceil(N/128)/4) above 2^31-1; all checked
 * before any launch), TARA_ERR_CUDA (workspace allocation or launch failure).             */
int tara_attn_forward(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                      const tara_token_meta* meta, const tara_params* p,
                      tara_tensor* O, float* LSE, void* stream);

/* ---- host buffers ------------------------------------------------------------------------ */
/* The same operation with Q, K, V, O, LSE and every metadata array (seg, time_s, pic, m,
 * extra_m) in HOST memory; pinned memory (cudaHostAlloc / cudaHostRegister) lets the copies
 * overlap the kernels, pageable memory works but serialises them.  The pages have no
 * counterpart: it is the runtime around the kernel for callers whose tensors live on the host.
 *   The B*H (branch, head) planes are processed in chunks of consecutive planes (at most about
 *   1 GiB of Q, K, V and O each, within one branch when the metadata is per branch; 1, 2, 4,
 *   ... planes at the start and the same ramp reversed at the end): per chunk, the
 *   host->device copies of Q, K, V run on one internal stream, the attention (the kernels of
 *   tara_attn_forward on device chunk buffers) on one of two internal compute streams, and the
 *   device->host copies of O and LSE on a fourth.  Two chunk buffer sets, each with its own
 *   workspace, and the two compute streams alternate between consecutive chunks, so transfers
 *   overlap kernels and one chunk's kernel fills the SMs the previous one's last wave leaves.
 *   Ordering: everything runs after the work already queued on `stream`, and `stream` waits
 *   for the last copy; the call itself does not block the host.  The host buffers must stay
 *   valid and unmodified until `stream` has completed (as with cudaMemcpyAsync).
 *   Device memory: the metadata plus two chunk sets with their workspaces, cached per device
 *   and grown with cudaMalloc (a growth synchronises the device).  A kernel-event pair pending for the
 *   calling thread (tara_set_kernel_events) is dropped.
 * Same arguments and checks as tara_attn_forward (shapes, dtypes, parameters, extra
 * bindings) except that pointers are host pointers with no alignment requirement.
 * Errors: TARA_ERR_NULL, _SHAPE, _DTYPE, _HEAD_DIM, _PARAM, _ALIGN, _TOO_LARGE, TARA_ERR_CUDA;
 * an error after the first copy was queued still leaves `stream` waiting for the queued work. */
int tara_attn_forward_host(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                           const tara_token_meta* meta, const tara_params* p,
                           tara_tensor* O, float* LSE, void* stream);

/* ---- 8-bit quantisation of Q and K ------------------------------------------------------ */
/* The quantisation tara_attn_forward runs when p->qk_int8 = 1, exposed for callers that keep
 * the codes ("TARA: ...", "Three backends" names dense INT8 kernels without their scaling;
 * the scheme below is this library's reading).
 *   Q, K    : device tensors [B][H][N][D], bf16 or fp16, D = 64 or 128, same shape and dtype,
 *             finite values, 16-byte aligned.
 *   q_codes : device int8 [B][H][N][D] (written): Q quantised per token.
 *   q_scale : device float [B][H][N] (written).
 *   k_codes : device int8 [B][H][N][D] (written): K quantised per block of 128 consecutive
 *             tokens of one (branch, head); the last block holds the N % 128 remaining tokens.
 *   k_scale : device float [B][H][ceil(N/128)] (written).
 *   stream  : CUDA stream, 0 for the legacy default stream.
 * Per group: amax = max |x|, inv = 127 / amax, code = rint(x * inv) (float32 product, ties to
 * even), scale = amax / 127 (IEEE float32 divisions); amax <= 1e-30 gives codes 0, scale 0.
 * x is approximated by code * scale.  Code arrays 16-byte aligned, scale arrays 4-byte.
 * Errors: TARA_ERR_NULL, _SHAPE, _DTYPE, _HEAD_DIM, _ALIGN, _TOO_LARGE before any launch;
 * TARA_ERR_CUDA on a launch failure.                                                       */
int tara_quantize_qk_int8(const tara_tensor* Q, const tara_tensor* K, int8_t* q_codes,
                          float* q_scale, int8_t* k_codes, float* k_scale, void* stream);

/* ---- allocation-free variant ------------------------------------------------------------ */
/* Largest scratch (bytes) tara_attn_forward_noalloc can use: per metadata set and 128-token
 * tile, two copies (ascending and descending tile order) of a 32-byte tile record and of
 * 128 16-byte key records, 4,160 bytes (8 MiB covers one shared set of up to ~258,000
 * tokens).  The array is part of the loaded module: every device that loads the library
 * holds it until the process exits.                                                       */
#define TARA_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Same operation, arguments and checks as tara_attn_forward for bf16/fp16 inputs, but it
 * never allocates: no cudaMalloc, no cudaFree, no allocating library call.  It is meant for
 * callers that cannot allocate device memory while they run (frameworks that own all device
 * memory through their own pool, serving loops that must not stall in the allocator).  The
 * pages have no counterpart to this entry point.
 *   - Scratch: a fixed module array of TARA_NOALLOC_SCRATCH_BYTES on each device instead of
 *     the cached workspace; sizes that need more return TARA_ERR_TOO_LARGE before anything
 *     is launched.  fp32 inputs return TARA_ERR_DTYPE (their kernel needs no scratch; call
 *     tara_attn_forward); qk_int8 = 1 returns TARA_ERR_PARAM (its 8-bit copies of Q and K
 *     do not fit the array).
 *   - Set-up: the first call on each device (that device current) looks up the array's device
 *     address with cudaGetSymbolAddress; make that first call before any stream capture.
 *   - Sharing: every call on a device uses the same array and leaves its contents behind;
 *     calls never read what an earlier call left (each call rewrites every record it reads).
 *     Calls whose work overlaps on the GPU (different streams, or concurrent with each other)
 *     race on the array: serialise them on one stream.
 *   - Timing: a CUDA-event pair armed with tara_set_kernel_events brackets its attention
 *     kernel, as for tara_attn_forward.                                                   */
int tara_attn_forward_noalloc(const tara_tensor* Q, const tara_tensor* K, const tara_tensor* V,
                              const tara_token_meta* meta, const tara_params* p,
                              tara_tensor* O, float* LSE, void* stream);

/* Profiling hook: the next tara_attn_forward call made by this host thread records the CUDA
 * event `start` on its stream immediately before launching its attention kernel and `stop`
 * immediately after it (the tile-summary kernel is outside the pair).  Both are cudaEvent_t
 * handles created by the caller; NULL for both clears a pending pair.  The pair is used once.
 * Returns TARA_OK, or TARA_ERR_NULL when exactly one of the two is NULL.                   */
int tara_set_kernel_events(void* start, void* stop);

/* Every kernel bounds each of its waits.  A kernel that gives up sets a per-device status
 * word and returns early (its outputs are then unspecified); while the word is set, later
 * attention launches on that device skip their work as well.  This call synchronises
 * `stream`, returns TARA_ERR_DEVICE_TIMEOUT if the word is set (and clears it), TARA_ERR_CUDA
 * if the synchronisation failed, TARA_OK otherwise.                                       */
int tara_device_status(void* stream);

/* Debug build.  The library can be compiled with -DTARA_DEBUG=1 (python -m
 * video_diffusion_attention_b200.build --debug writes libtara_attn_debug.so beside the release
 * library).  Its kernels then check on the device what the host cannot see: that target and
 * guide tokens carry finite times and target tokens finite mask weights, and that every row,
 * plane and output index they derive stays inside its array.  A failed check records itself
 * in the status word, the checked access is skipped and nothing traps; tara_device_status
 * then returns TARA_ERR_DEBUG_CHECK (and clears the word).  The release build has no such
 * checks.  Returns 1 in the debug build, 0 otherwise.  The pages have no counterpart.     */
int tara_debug_build(void);

/* Self-test of that machinery (failure detection without faulting the GPU): launches one
 * warp on `stream` that waits on a shared-memory barrier with a limit of limit_us
 * microseconds (1..10^7).  With arrive == 0 nothing ever arrives, so the wait gives up and
 * sets the status word, which the next tara_device_status reports; with arrive != 0 the
 * barrier completes and nothing is set.  Returns TARA_ERR_PARAM for a limit out of range,
 * TARA_ERR_CUDA on a launch failure, TARA_OK otherwise.  The pages have no counterpart.   */
int tara_selftest_wait(int limit_us, int arrive, void* stream);

/* ---- target-mask preparation (device) -------------------------------------------------- */
/* Turns a soft pixel mask into the per-target-token weights m the forward pass reads
 * ("BFS H3 Reference Attention Binding (Experimental)", "The exact rule": soft masks are
 * area-downsampled to the target's patch resolution and averaged across the latent temporal
 * spans; "Inputs you'll set": one static mask or one mask per prepared shot frame;
 * "Common issues": any other mask length is an error).
 *   mask              : device float array [F_in][Hp][Wp], row-major, values normally in [0,1]
 *   F_in              : 1 (static mask) or shot_len (one mask per frame of the prepared shot)
 *   shot_len          : frames of the prepared shot; must be 17n+5 (n >= 0)
 *   frames_per_latent : tau, pixel frames per latent frame; latent frame f averages frames
 *                       [f*tau, min((f+1)*tau, shot_len))
 *   F_lat, Hq, Wq     : latent frames and patch grid of the target video
 *   m_out             : device float array [F_lat][Hq][Wq] (written), i.e. the target
 *                       tokens' m in packing order (frame-major, row-major patches)
 * Cell (y, x) of a frame is the exact area average of the pixel image over
 * [y*Hp/Hq, (y+1)*Hp/Hq) x [x*Wp/Wq, (x+1)*Wp/Wq).  A static mask is copied to every latent
 * frame.  Errors: TARA_ERR_NULL, TARA_ERR_SHAPE (a size < 1, or latent frames beyond the
 * shot), TARA_ERR_MASK_LENGTH, TARA_ERR_TOO_LARGE (F_lat > 65535 or Wq > 12288),
 * TARA_ERR_ALIGN (4 bytes),
 * TARA_ERR_CUDA; checked before launching.  Asynchronous on `stream`.                    */
int tara_prepare_target_mask(const float* mask, int32_t F_in, int32_t Hp, int32_t Wp,
                             int32_t shot_len, int32_t frames_per_latent, int32_t F_lat,
                             int32_t Hq, int32_t Wq, float* m_out, void* stream);

/* ---- the token-metadata packer (host) ------------------------------------------------- */
/* One segment of the packed joint sequence, in packing order.  A segment is `frames` latent
 * frames of `tokens_per_frame` tokens each (text, pictures and audio use frames = 1).
 * Token (f, p) of a segment (frame f, patch p in row-major patch order) gets
 *   seg    = kind
 *   time_s = (float)(t0_s + f * frame_dt_s)       evaluated in double, rounded once
 *   pic    = pic for PICTURE segments (must be 1..9), 0 otherwise
 *   m      = mask value for TARGET segments: 1 if mask_len == 0 (no mask: the gain applies to
 *            the whole output video); mask[p] if mask_len == tokens_per_frame (one static
 *            mask); mask[f*tokens_per_frame + p] if mask_len == frames*tokens_per_frame (one
 *            mask per frame); 1 for every non-TARGET token.
 * ("BFS H3 Reference Attention Binding", "Inputs you'll set": no mask, one static mask, or
 * one mask per prepared shot frame; the mask is taken here already at patch resolution.)   */
typedef struct {
  int32_t      kind;              /* tara_seg                                               */
  int32_t      frames;            /* >= 1                                                   */
  int32_t      tokens_per_frame;  /* >= 1                                                   */
  int32_t      pic;               /* PICTURE: 1..9; ignored otherwise                       */
  double       t0_s;              /* time of frame 0 on the shared clock                    */
  double       frame_dt_s;        /* seconds per latent frame (e.g. 4/24)                   */
  const float* mask;              /* host array, TARGET only; may be NULL if mask_len == 0  */
  int64_t      mask_len;
} tara_segment;

/* Total token count of a segment list (>= 0), or a negative status on a bad list. */
int64_t tara_packed_length(const tara_segment* segs, int32_t n_segs);

/* Write the four metadata arrays (host memory, capacity N each) for the segment list.
 * Returns TARA_ERR_NULL, TARA_ERR_SEGMENT (kind > 5, frames or tokens_per_frame < 1, PICTURE
 * without pic in 1..9, mask_len not in {0, tokens_per_frame, frames*tokens_per_frame}, or a
 * non-finite time), TARA_ERR_CAPACITY (N != total length) or TARA_OK.  Nothing is written
 * unless the whole list is valid.                                                         */
int tara_pack_token_meta(const tara_segment* segs, int32_t n_segs,
                         uint8_t* seg, float* time_s, uint8_t* pic, float* m, int32_t N);

#ifdef __cplusplus
}
#endif

#endif /* TARA_ATTN_H_ */
