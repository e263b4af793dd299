/*
 * wam.h - C ABI of the B200 (sm_100a) attention stack of one world-action-model action chunk.
 *
 * The stack has three parts, each defined on the pages named below:
 *   (a) block-causal video prefill of a per-layer K/V cache over history frames and imagined
 *       future frames denoised to sigma* ("Long-WAM 源码精读" §03-§04: the video expert rolls the
 *       future latents from pure noise to sigma* = 0.9 in 4 steps, then prefill_video_cache
 *       builds a per-layer {"k","v"} list; "Long-WAM: Scaling the Context of World-Action
 *       Models | Summary" §3.1-3.2: video queries read their own and earlier visual blocks);
 *   (b) Interval KV-Fusion ("世界模型之Faster-WAM详解" §3.3: the K/V of one depth interval are
 *       folded into one K/V pair of one layer's length with softmax-normalised weights);
 *   (c) asymmetric action attention inside the flow-matching Euler loop ("Fast-WAM 精读"
 *       SECTION 07: K = [K_video; K_action], V = [V_video; V_action], Q/K/V of the actions
 *       recomputed every step; Long-WAM Summary §4.2: one online softmax over the two buffers).
 *
 * Conventions shared by every entry point
 *   - Tensors are token-major [B, tokens, H, D], contiguous, as on "Fast-WAM 精读" SECTION 04
 *     ([N, 24, 128] per episode).  A per-layer cache or fused cache holds all N = F*T tokens.
 *   - Device pointers are caller-owned.  The library never allocates, frees or synchronises
 *     device memory, and never keeps a pointer after a call returns.
 *   - Every call that touches the GPU is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and returns once its kernels are enqueued.
 *   - Every call returns a wam_status; nothing throws or aborts across the ABI.  On an error
 *     the arguments are rejected before anything is launched, and wam_last_error() returns a
 *     message for the calling thread.
 *   - Frame padding and attention blocks are HOST arrays: the host knows which history frames
 *     exist, and the library turns them into per-launch work lists (no device mask is read).
 *   - Supported: dtype WAM_F32 or WAM_BF16; D in {64, 128}; 1 <= T; 1 <= F <= WAM_MAX_FRAMES;
 *     B * F <= WAM_MAX_EPISODE_FRAMES.  bf16 with D = 128 and T % 128 == 0 runs on the tensor
 *     cores; every other supported shape runs the fp32-accumulating CUDA-core path (also on
 *     the GPU).  Anything else returns WAM_ERR_UNSUPPORTED.
 *   - Pointers to bf16 or fp32 tensors must be 16-byte aligned.
 */
#ifndef WAM_H_
#define WAM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* wam_stream_t; /* the same handle as cudaStream_t */

#define WAM_MAX_FRAMES 256
#define WAM_MAX_EPISODE_FRAMES 1024
#define WAM_MAX_FUSE_LAYERS 16
#define WAM_MAX_COPY_TENSORS 128
#define WAM_MAX_NVFP4_TENSORS 64

typedef enum {
  WAM_OK = 0,
  WAM_ERR_INVALID_ARGUMENT = 1, /* a null pointer, bad size, misaligned pointer, bad range */
  WAM_ERR_UNSUPPORTED = 2,      /* a valid request the library has no kernel for */
  WAM_ERR_CUDA = 3,             /* a CUDA runtime error while configuring or launching */
  WAM_ERR_WORKSPACE = 4,        /* a workspace that is missing or too small */
  WAM_ERR_TIMEOUT = 5           /* a bounded device-side wait gave up (wam_device_error) */
} wam_status;

typedef enum { WAM_F32 = 0, WAM_BF16 = 1 } wam_dtype;

/*
 * Geometry shared by the video and action calls.
 *   B episodes, H heads, D head dim, T tokens per latent frame, F = history + imagined frames;
 *   token t belongs to frame t / T, and a cache holds N = F * T tokens.
 *   frame_pad   host uint8 [B, F], 1 = padding frame (unavailable early history, Long-WAM
 *               Summary §3.3), NULL = no padding.  Keys of padding frames are never read;
 *               queries of padding frames are not computed and their output rows are not
 *               written; their K/V are neither stored nor fused (those rows keep their
 *               previous contents).
 *   frame_block host int32 [F], nondecreasing attention-block id of each frame, NULL = one
 *               block per frame.  A video query reads keys whose block id is <= its own
 *               (Long-WAM Summary §3.1-3.2); grouping imagined frames into one block lets
 *               future slots read each other (Faster-WAM详解 §3.1).
 */
typedef struct {
  int32_t B, H, D, T, F;
  const uint8_t* frame_pad;
  const int32_t* frame_block;
} wam_video_layout;

/*
 * Interval KV-Fusion folded into the cache write of one layer (Faster-WAM详解 §3.3):
 * for the stored (non-padding) frames of the call,
 *   first_in_interval:  acc  = w * K_j               (acc is not read)
 *   middle layers:      acc += w * K_j
 *   last_in_interval:   fused = round(acc + w * K_j) (acc is read, not written)
 * and the same for V.  A one-layer interval sets both flags.  acc_k/acc_v are caller-owned
 * fp32 device scratch [B, N, H, D]; fused_k/fused_v are device [B, N, H, D] of the call's dtype.
 * The fold runs inside the prefill kernel from the call's own K/V input (middle layers add
 * into acc by L2 reductions), so the stored per-layer cache is never re-read for fusion.
 * Calls that use the same accumulator must not overlap on the GPU.
 */
typedef struct {
  float weight;
  int32_t first_in_interval;
  int32_t last_in_interval;
  float* acc_k;
  float* acc_v;
  void* fused_k;
  void* fused_v;
} wam_fuse_epilogue;

/*
 * Block-causal video attention of one layer for the query frames [f_begin, f_end), with the
 * store of their K/V into that layer's cache ("Long-WAM 源码精读" §04 prefill_video_cache;
 * Long-WAM Summary §3.2, §4.2 observed-video KV computed once and reused).
 *
 *   q, k_new, v_new  device [B, (f_end - f_begin) * T, H, D], dtype dt
 *   k_cache, v_cache device [B, N, H, D], dtype dt.  Keys of frames [0, f_begin) are read
 *                    from here (frames stored by earlier calls); if store_kv != 0 the
 *                    non-padding frames of [f_begin, f_end) are written here from k_new/v_new.
 *                    May be NULL when f_begin == 0 and store_kv == 0.
 *   o                device [B, (f_end - f_begin) * T, H, D], dtype o_dt (WAM_F32 or dt);
 *                    O_q = sum_k softmax_k(q.k / sqrt(D)) v_k over the allowed keys; rows of
 *                    padding frames are left unwritten.
 *   fuse             NULL, or the fusion epilogue above (needs store semantics: the frames
 *                    folded are the non-padding frames of [f_begin, f_end)).
 * A call must not split an attention block: frame f_begin starts a block and f_end is F or
 * starts a block.  Accumulation is fp32; P is rounded to bf16 for the PV product on the
 * tensor-core path.
 */
wam_status wam_video_prefill_kv(const wam_video_layout* layout, wam_dtype dt,
                                int32_t f_begin, int32_t f_end,
                                const void* q, const void* k_new, const void* v_new,
                                void* k_cache, void* v_cache, int32_t store_kv,
                                void* o, wam_dtype o_dt,
                                const wam_fuse_epilogue* fuse, wam_stream_t stream);

/*
 * Standalone Interval KV-Fusion (Faster-WAM详解 §3.3): for the non-padding frames of
 * [f_begin, f_end), fused = round(sum_j weights[j] * layer_j) computed in fp32, for K and V.
 *   k_layers, v_layers host arrays of n_layers device pointers [B, N, H, D] (dtype dt)
 *   weights            host float [n_layers] (softmax-normalised, see wam_fuse_weights)
 *   fused_k, fused_v   device [B, N, H, D] (dtype dt); padding frames are not written.
 * 1 <= n_layers <= WAM_MAX_FUSE_LAYERS.
 */
wam_status wam_fuse_interval_kv(const wam_video_layout* layout, wam_dtype dt, int32_t n_layers,
                                const void* const* k_layers, const void* const* v_layers,
                                const float* weights, int32_t f_begin, int32_t f_end,
                                void* fused_k, void* fused_v, wam_stream_t stream);

/*
 * Asymmetric action attention of one action-expert layer at one Euler step ("Fast-WAM 精读"
 * SECTION 07; Long-WAM Summary §3.2, §4.2; Faster-WAM详解 §3.2 SparseMoT):
 *   O = softmax(Q_a [K_video(non-padding frames); K_a]^T / sqrt(D)) [V_video; V_a]
 * computed as split-KV partials over the video keys and the action buffer, merged by one
 * shared online-softmax normalisation (no concatenated buffer is formed).
 *   fused_k, fused_v device [B, N, H, D] (dtype dt), or both NULL for a layer outside the
 *                    interaction set (action self-attention only)
 *   qa, ka, va       device [B, n_act, H, D] (dtype dt), 1 <= n_act <= 128
 *   o                device [B, n_act, H, D], dtype o_dt (WAM_F32 or dt)
 *   workspace        device scratch of at least wam_action_attn_workspace_size() bytes, 16-byte
 *                    aligned, zero-filled before its first use.  Its first 64 KiB hold one
 *                    arrival ticket per (episode, head) (B * H <= 16384); every call that
 *                    completes leaves them at zero, so one workspace serves calls of any layout
 *                    in turn.  Calls that share a workspace must not overlap on the GPU.  May be
 *                    NULL when the size is 0.  (The tensor-core read of 128-key tiles,
 *                    T % 128 == 0, merges its partials on chip and leaves the workspace
 *                    untouched; the size query does not depend on which path will run.)
 * Action tokens attend to each other bidirectionally.  Returns WAM_ERR_WORKSPACE if the
 * workspace is missing or too small.
 */
wam_status wam_action_attn(const wam_video_layout* layout, wam_dtype dt,
                           const void* fused_k, const void* fused_v,
                           int32_t n_act, const void* qa, const void* ka, const void* va,
                           void* o, wam_dtype o_dt, void* workspace, size_t ws_bytes,
                           wam_stream_t stream);

/*
 * wam_action_attn with flags (0: the same call).
 *   WAM_ACTION_FUSED_READY  the caller guarantees that the fused pair is not written by the call
 *                           issued on `stream` right before this one.  In the action loop the
 *                           fused cache is read-only (the video stage completed it), and the
 *                           read may then start loading its fused tiles while that call is still
 *                           running (programmatic dependent launch); the action Q/K/V are read
 *                           only after it has completed.  Used by the tensor-core read of 128-key
 *                           tiles; the other paths ignore it.
 * Unknown flag bits return WAM_ERR_INVALID_ARGUMENT.
 */
#define WAM_ACTION_FUSED_READY 1u
wam_status wam_action_attn_ex(const wam_video_layout* layout, wam_dtype dt,
                              const void* fused_k, const void* fused_v,
                              int32_t n_act, const void* qa, const void* ka, const void* va,
                              void* o, wam_dtype o_dt, void* workspace, size_t ws_bytes,
                              uint32_t flags, wam_stream_t stream);

/*
 * Bytes of workspace wam_action_attn needs for this layout on the current device
 * (with_video != 0: a layer that reads a fused pair).  Depends on the device's SM count.
 */
wam_status wam_action_attn_workspace_size(const wam_video_layout* layout, wam_dtype dt,
                                          int32_t n_act, int32_t with_video, size_t* bytes);

/*
 * One Euler step of the flow-matching sampler, x <- x + dsigma * v, elementwise over n fp32
 * values ("Long-WAM 源码精读" §03: path x_s = (1-s) x + s eps, target u = eps - x;
 * "Fast-WAM 精读" SECTION 07: the scheduler updates the action latent each step).
 *   x device fp32 [n], updated in place; v device fp32 [n]; dsigma = sigma_{i+1} - sigma_i.
 */
wam_status wam_flow_euler_step(int64_t n, float* x, const float* v, float dsigma,
                               wam_stream_t stream);

/*
 * Move whole frames of per-layer K/V tensors from one buffer set to another, for a history
 * window kept across chunks ("Long-WAM ... | Summary" §4.2: the observed-video K/V is
 * computed once and reused; one frame arrives per chunk, so the window slides and every kept
 * frame moves to an earlier position).  For each pair j < n and every episode b:
 *   dst[j][b, (f_dst + i) * T + t, :, :] = src[j][b, (f_src + i) * T + t, :, :]
 *   for 0 <= i < n_frames, 0 <= t < T.
 *   src, dst  host arrays of n device pointers [B, F*T, H, D] (dtype dt), 16-byte aligned;
 *             src[j] and dst[j] must not overlap (keep the window in two buffer sets used in
 *             turn).  1 <= n <= WAM_MAX_COPY_TENSORS.
 *   frames    0 <= f_src, f_dst and f_src + n_frames, f_dst + n_frames <= F; n_frames == 0
 *             launches nothing.
 * Padding is not consulted: whole frames are copied.
 */
wam_status wam_copy_frames(const wam_video_layout* layout, wam_dtype dt, int32_t n,
                           const void* const* src, void* const* dst, int32_t f_src,
                           int32_t f_dst, int32_t n_frames, wam_stream_t stream);

/*
 * wam_video_prefill_kv with the fusion epilogue, for callers that cannot allocate device memory
 * (no counterpart on the pages: it is a deployment convenience of this library).
 *
 * The epilogue's fp32 accumulator normally comes from the caller (wam_fuse_epilogue.acc_k /
 * acc_v).  Code that runs while a CUDA graph is being captured, plug-ins that get a fixed
 * memory pool from their host, or runtimes that allocate everything up front cannot call
 * cudaMalloc for it.  This entry point keeps the accumulator in a device array inside the
 * library instead; the caller passes only inputs and outputs.  Arguments are those of
 * wam_video_prefill_kv, with the epilogue given as weight / first / last / fused_k / fused_v.
 *   - Limit: B * F * T * H * D <= WAM_NOALLOC_FUSE_ACC_ELEMS (about 4.2 million elements, for
 *     K and for V); larger layouts return WAM_ERR_UNSUPPORTED and launch nothing.  The array
 *     (2 x 16 MiB) is held on every GPU that loads the library until the process exits.
 *   - Every call looks the array's address up on the current device (cudaGetSymbolAddress,
 *     which allocates nothing).  The first call on a device may also load the library's
 *     device code there: make that first call before any stream capture.
 *   - A one-layer interval (first_in_interval and last_in_interval) never touches the array
 *     and is not held to the limit.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - Every call shares the one array, which keeps what the last call left in it: a middle or
 *     last call of an interval reads what the previous call of that interval accumulated, and
 *     a first call overwrites it (nothing has to start at zero).  Calls that overlap on the
 *     GPU (other streams, other threads) race on it; keep them ordered.
 */
#define WAM_NOALLOC_FUSE_ACC_ELEMS (4 * 1024 * 1024)
wam_status wam_video_prefill_kv_fuse_noalloc(const wam_video_layout* layout, wam_dtype dt,
                                             int32_t f_begin, int32_t f_end,
                                             const void* q, const void* k_new, const void* v_new,
                                             void* k_cache, void* v_cache, int32_t store_kv,
                                             void* o, wam_dtype o_dt,
                                             float weight, int32_t first_in_interval,
                                             int32_t last_in_interval,
                                             void* fused_k, void* fused_v, wam_stream_t stream);

/*
 * Low-precision fused cache: NVFP4 encoding of fused K or V tensors ("Long-WAM: 机器人操作模型
 * 的长历史..." §四: the LongLive-2.0 stack keeps its KV cache block-wise in NVFP4, about 3.6x
 * smaller; "Long-WAM ... | Summary" §4.2: Long-WAM itself keeps BF16).  The pages name the
 * format, not its parameters; this library takes NVIDIA's public NVFP4:
 *   elements E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one E4M3 scale per 16 consecutive
 *   elements along D, one fp32 scale per tensor s_g = amax / (6 * 448) over the tensor's
 *   non-padding frames; x ~ e2m1 * e4m3 * s_g.  Codes are chosen in fp32 (IEEE division and
 *   products), rounded to nearest even and saturated; zero takes the +0 code.
 *   fused   host array of n device pointers, bf16 [B, N, H, D] (the stored fused pairs)
 *   codes   host array of n device pointers, uint8 [B, H, N, D / 2]: head-major (one 128-key
 *           tile of one head is one contiguous run), element 2i in the low nibble of byte i
 *   scales  host array of n device pointers, uint8 [B, H, N, D / 16]: E4M3 codes
 *   s_g     device float [n]: each tensor's scale
 *   workspace device scratch of wam_nvfp4_workspace_size(n) bytes, 16-byte aligned
 * Rows of padding frames are not read and their codes and scales are not written.  Two kernels
 * on `stream`; 1 <= n <= WAM_MAX_NVFP4_TENSORS; D % 16 == 0 (D in {64, 128}); bf16 only.
 */
wam_status wam_nvfp4_workspace_size(int32_t n, size_t* bytes);
wam_status wam_fused_to_nvfp4(const wam_video_layout* layout, int32_t n, const void* const* fused,
                              void* const* codes, void* const* scales, float* s_g,
                              void* workspace, size_t ws_bytes, wam_stream_t stream);

/*
 * The asymmetric action read of wam_action_attn over an NVFP4 fused pair (as wam_fused_to_nvfp4
 * writes it): O = softmax(Q_a [K_video; K_a]^T / sqrt(D)) [V_video; V_a] with the video keys and
 * values taken as their decoded values e2m1 * e4m3 * s_g.
 *   k_codes, k_scales, v_codes, v_scales  device [B, H, N, 64] and [B, H, N, 8] (D = 128)
 *   k_sg, v_sg   device float: the tensors' scales (4-byte aligned)
 *   qa, ka, va   device bf16 [B, n_act, H, 128], 1 <= n_act <= 32; o device [B, n_act, H, 128]
 *                (o_dt WAM_F32 or WAM_BF16)
 *   workspace    as for wam_action_attn (wam_action_attn_workspace_size with dt = WAM_BF16)
 *   flags        0 or WAM_ACTION_FUSED_READY (as for wam_action_attn_ex: the codes and scales
 *                are not written by the call issued on `stream` right before this one)
 * T % 128 == 0.  The tiles are decoded exactly into fp16 and the matrix products run on fp16
 * operands with fp32 accumulation (the action Q/K/V are rounded to fp16 once: they must lie
 * within fp16's range, |x| < 65504); P is carried as two fp16 terms.
 */
wam_status wam_action_attn_nvfp4(const wam_video_layout* layout, const void* k_codes,
                                 const void* k_scales, const float* k_sg, const void* v_codes,
                                 const void* v_scales, const float* v_sg, int32_t n_act,
                                 const void* qa, const void* ka, const void* va, void* o,
                                 wam_dtype o_dt, void* workspace, size_t ws_bytes,
                                 uint32_t flags, wam_stream_t stream);

/* ---- host helpers (no GPU work) ---------------------------------------------------------- */

/*
 * Noise levels of an n-step sampler into host double sigmas[n_steps + 1]:
 *   u_i = (n - i) / n,  sigma_i = sigma_end + (1 - sigma_end) * phi(u_i)
 * phi(u) = shift * u / (1 + (shift - 1) u) (identity at shift = 1).  sigma_0 = 1 and
 * sigma_n = sigma_end exactly ("Long-WAM 源码精读" §04: linspace(1, 0, steps + 1), warped,
 * then rescaled so the end lands exactly on sigma* and the start stays pure noise).
 */
wam_status wam_flow_schedule(int32_t n_steps, double sigma_end, double shift, double* sigmas);

/* Softmax of n host logits into host weights (Faster-WAM详解 §3.3, W_fuse normalisation). */
wam_status wam_fuse_weights(int32_t n, const float* logits, float* weights);

/*
 * The video predicate the prefill kernels apply, written out per element for inspection:
 * mask[b, i, k] = 1 if query token f_begin*T + i may read key token k (k < f_end * T), else 0.
 *   mask device uint8 [B, (f_end - f_begin) * T, f_end * T].
 */
wam_status wam_debug_video_mask(const wam_video_layout* layout, int32_t f_begin, int32_t f_end,
                                uint8_t* mask, wam_stream_t stream);

/*
 * The work items of a bf16, D = 128 tensor-core prefill call over frames [f_begin, f_end)
 * (T % 128 == 0), in the order the call launches them on a device with n_sms SMs; host only,
 * no GPU needed.  An item is one valid query frame of one episode with the number of valid
 * key frames it reads; it runs as ceil(T / 256) x H consecutive CTAs, one resident per SM.
 * The order starts from longest first; each class of equal key-frame count is also tried right
 * behind the longest class and at the end, every candidate is scored by replaying in-order
 * dispatch of its CTAs onto n_sms SMs (cost per CTA: key tiles + 5), and the cheapest is
 * kept (longest first on ties; n_sms <= 0, or a single wave, keeps longest first).  A single
 * wave whose frames hold an even number of 128-row query tiles, and whose episodes each hold
 * an even number of items of unequal key-frame counts, is instead paired: within each
 * episode the items with most and fewest key frames become items 2i and 2i + 1, and each CTA
 * of a pair takes the same query tile of both frames (T / 128 x H CTAs per pair).
 *   episode, frame, n_key_frames: host int32 arrays with room for B * (f_end - f_begin);
 *   *n_items receives the number of items written; *paired (may be NULL) receives 1 for a
 *   paired order, else 0.
 */
wam_status wam_debug_prefill_order(const wam_video_layout* layout, int32_t f_begin, int32_t f_end,
                                   int32_t n_sms, int32_t* episode, int32_t* frame,
                                   int32_t* n_key_frames, int32_t* n_items, int32_t* paired);

/*
 * Failure-detection check: launches one warp that waits on a shared-memory mbarrier nothing
 * arrives on, giving up after `polls` polls (1 <= polls <= 2^24, the attention kernels'
 * own limit), and then records WAM_ERR_TIMEOUT in the device error word exactly as an
 * attention kernel does when one of its bounded waits gives up.  The kernel holds no TMA,
 * tensor-core or tensor-memory work and returns normally; wam_device_error() then reports
 * the timeout, and the device stays usable.  Asynchronous on `stream`.
 */
wam_status wam_debug_wait_timeout(int32_t polls, wam_stream_t stream);

/*
 * The work split of the NVFP4 read (T % 128 == 0) on a device with n_sms SMs; host only, no GPU
 * needed.  Every head of episode b is cut into kparts[b] parts at the same tile boundaries:
 * part r of k reads the video tiles [1 + r nv / k, 1 + (r + 1) nv / k) of the (episode, head)
 * (nv = 128-key tiles of the episode's valid frames) and part 0 also the action tile.  The
 * smallest part size is chosen for which all B * H * k CTAs fit in n_sms (one part per head if
 * none does).
 *   kparts host int32 [B]; *n_ctas the CTAs launched; *max_parts the largest kparts[b].
 */
wam_status wam_debug_action_plan(const wam_video_layout* layout, int32_t n_sms, int32_t* kparts,
                                 int32_t* n_ctas, int32_t* max_parts);

/*
 * Synchronise the current device and report its error word: WAM_OK, or WAM_ERR_TIMEOUT when
 * a kernel's bounded wait on an mbarrier gave up (the kernel then skipped its remaining work
 * and returned without faulting).  clear != 0 resets the word.  Host-blocking.
 */
wam_status wam_device_error(int32_t clear);

/* Thread-local message of the last failing call on this thread ("" if none). */
const char* wam_last_error(void);

/* ABI version of the library: major * 10000 + minor * 100 + patch. */
int32_t wam_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WAM_H_ */
