/*
 * dit.h — C ABI of the B200 (sm_100a) DiT denoiser forward library.
 *
 * The library computes one evaluation of the Diffusion Transformer denoiser
 * (the noise / covariance or velocity predictor of a latent diffusion or
 * rectified-flow model) on one GPU:
 *
 *   patchify + linear embed (+ 2D sin-cos positions)            "확산 트랜스포머"
 *     (itwiki.kr), section "잠재 공간과 패치화": T = (I/p)^2 tokens of width d;
 *   c = MLP(sinusoid(t)) + e(y)                                  same page, "adaLN-Zero":
 *     c is the sum of the timestep and class embeddings (or a pooled text vector);
 *   N blocks of  x += a1 * Attn(LN(x)(1+g1)+b1),  x += a2 * FFN(LN(x)(1+g2)+b2)
 *     with (b1,g1,a1,b2,g2,a2) = Linear(SiLU(c))                 same page, "adaLN-Zero";
 *   final modulated LN, linear decoder to p x p x 2C per token, unpatchify
 *                                                                "Sora / DiT" (cv-learn.com),
 *     "방법 및 아키텍처"; itwiki page, "잠재 공간과 패치화";
 *   classifier-free guidance  e = e(null) + s (e(c) - e(null))   "Sora / DiT", guidance bullet;
 *   video variant: spacetime patches, QK-RMSNorm and 3D RoPE, velocity head
 *                                                                "GOKU : Flow Based Video
 *     Generative Foundation Models" (blog.outta.ai), sections 2.2 and 2.3;
 *   and the sampler update around it (dit_sampler_step, dit_sample): a deterministic
 *     step of the DDPM forward process x_t = sqrt(abar_t) x_0 + sqrt(1-abar_t) eps
 *     ("Sora / DiT", training-objective bullet) or an Euler step of the rectified-flow
 *     path x_t = t x_1 + (1-t) x_0 ("GOKU", section 2.3).
 *
 * Conventions for every entry point:
 *   - Pointers named "dev" are CUDA device pointers on the current device; "host"
 *     pointers are ordinary (preferably pinned) host memory.
 *   - All floating-point I/O is float32 (IEEE binary32); labels are int32.
 *   - Work is enqueued on the given cudaStream_t (0 = legacy default stream) and
 *     the call returns without waiting unless stated otherwise.
 *   - A dit_status is returned; DIT_OK (0) means the work was enqueued.  Errors
 *     found on the host return before anything is launched.  Errors found on
 *     the device (a label outside [0, num_classes], a bounded wait that ran out)
 *     are recorded in a per-handle device status word, read by dit_sync_status.
 *   - No entry point traps, aborts or waits without a bound.
 */
#ifndef DIT_B200_H
#define DIT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dit_stream_t; /* same type as cudaStream_t */

typedef enum {
  DIT_OK = 0,
  DIT_ERR_INVALID_ARG = 1,    /* null pointer, bad size, batch > max_batch, bad weight count */
  DIT_ERR_UNSUPPORTED = 2,    /* shape the kernels do not cover (e.g. head dim not 64 or 72) */
  DIT_ERR_OOM = 3,            /* device allocation failed in dit_create */
  DIT_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
  DIT_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up (device status word) */
  DIT_ERR_BAD_LABEL = 6,      /* a class label outside [0, num_classes]; it was clamped */
  DIT_ERR_NO_DEVICE = 7       /* no sm_100 device is current */
} dit_status;

enum { DIT_DTYPE_F32 = 0, DIT_DTYPE_BF16 = 1 };
enum { DIT_POS_SINCOS2D = 0, DIT_POS_ROPE3D = 1 };
enum { DIT_COND_CLASS = 0, DIT_COND_VECTOR = 1 };
/* How the condition enters the blocks: the four designs "확산 트랜스포머" (itwiki.kr) compares
   in section "조건 주입 방식" (conditioning), and what each block computes:
   DIT_BLOCK_ADALN_ZERO  (b1,g1,a1,b2,g2,a2) = Linear(SiLU(c));
                         x += a1 Attn(LN(x)(1+g1)+b1);  x += a2 FFN(LN(x)(1+g2)+b2)
   DIT_BLOCK_IN_CONTEXT  e_t and e_y become two extra tokens in front of the patch tokens
                         (no position; removed after the last block); plain pre-norm blocks
                         x += Attn(LN1(x));  x += FFN(LN2(x)) with learned LN affines
   DIT_BLOCK_CROSS_ATTN  plain pre-norm blocks with a cross-attention sublayer after the
                         self-attention: x += CrossAttn(LNx(x), [e_t, e_y])
   DIT_BLOCK_ADALN       (b1,g1,b2,g2) = Linear(SiLU(c)); the adaLN-Zero block without gates
   (e_t = timestep MLP output, e_y = label row or text vector, c = e_t + e_y.)  The two
   unmodulated designs end with a learned-affine LayerNorm before the decoder, the two
   modulated ones with the adaLN (shift, scale) LayerNorm. */
enum { DIT_BLOCK_ADALN_ZERO = 0, DIT_BLOCK_IN_CONTEXT = 1, DIT_BLOCK_CROSS_ATTN = 2, DIT_BLOCK_ADALN = 3 };

/* Model and workload description.  Image models use frames = patch_t = 1. */
typedef struct dit_config {
  int dtype;          /* DIT_DTYPE_F32: float32 SIMT kernels; DIT_DTYPE_BF16: bf16 operands on
                         tcgen05 tensor cores with float32 accumulation, statistics and residual */
  int in_channels;    /* C of the latent (4 for the image models, 16 for the video model) */
  int frames, height, width;       /* latent extent F, H, W */
  int patch_t, patch_h, patch_w;   /* patch extent; each must divide the latent extent */
  int hidden;         /* d */
  int depth;          /* N blocks */
  int heads;          /* attention heads; head dim d/heads must be 64 or 72 */
  int mlp_hidden;     /* FFN width (4d in every DiT size) */
  int learn_sigma;    /* 1: decoder emits 2C channels (noise + diagonal covariance); 0: C */
  int pos_kind;       /* DIT_POS_SINCOS2D (added to tokens) or DIT_POS_ROPE3D (rotates q, k) */
  int qk_norm;        /* 1: RMSNorm with learnable gain on q and k of each head */
  int cond_kind;      /* DIT_COND_CLASS: label table of num_classes+1 rows (last = null);
                         DIT_COND_VECTOR: caller passes a float32 vector of width d per sample */
  int num_classes;    /* 1000 for ImageNet; the null label is num_classes */
  int freq_dim;       /* width of the timestep sinusoid (256; a multiple of 4, at most 1536) */
  int max_batch;      /* largest user batch B; device workspace is sized for 2*max_batch rows */
  float t_scale;      /* the sinusoid sees t * t_scale (1 for integer steps, 1000 for t in [0,1)) */
  int block_kind;     /* DIT_BLOCK_* (0 = adaLN-Zero, the design of the standard DiT models) */
  int ffn_fp8;        /* 1: the feed-forward matmuls run on FP8 E4M3 operands (bf16 path only):
                         fc1.w / fc2.w quantised per output channel (scale amax / 448) at create,
                         the LN output per token (amax / 448), the hidden activation per token with
                         the scale (||u||_2 max_n ||fc1.w_n||_2 + max |fc1.b|) / 448, a bound on
                         |GELU(z)| known before z is formed; accumulation stays float32 */
  int attn_fp8;       /* 1: the self-attention's in- and out-projection run on FP8 E4M3 operands
                         (bf16 path only): qkv.w / proj.w quantised per output channel (scale
                         amax / 448) at create, the LN output and the concatenated heads' output
                         per token (amax / 448); q, k, v, the attention itself and the residual
                         stream stay bf16 / float32 */
} dit_config;

typedef struct dit_handle dit_handle;

/*
 * dit_create — validate the configuration, allocate device weights and workspace,
 * upload and convert the weights.
 *
 * weights: n_weights host float32 arrays in this fixed order (linear weights are
 * row-major [out, in]; K_p = C*patch_t*patch_h*patch_w; P = patch_t*patch_h*patch_w*C_out):
 *   pe.w [d, K_p] (patch vector order c, i_t, i_h, i_w — a flattened Conv weight), pe.b [d],
 *   t.w1 [d, freq_dim], t.b1 [d], t.w2 [d, d], t.b2 [d],
 *   y.table [num_classes+1, d]                          (DIT_COND_CLASS only),
 *   for each block: ada.w [6d, d], ada.b [6d], qkv.w [3d, d], qkv.b [3d],
 *                   q_norm.g [d/heads], k_norm.g [d/heads]   (qk_norm only),
 *                   proj.w [d, d], proj.b [d], fc1.w [mlp, d], fc1.b [mlp],
 *                   fc2.w [d, mlp], fc2.b [d],
 *   final.ada.w [2d, d], final.ada.b [2d], dec.w [P, d], dec.b [P].
 * The ada.w output rows are ordered (shift1, scale1, gate1, shift2, scale2, gate2),
 * the final ones (shift, scale); qkv.w rows are [q | k | v], heads contiguous.
 * The other block designs change the per-block list and the final layer:
 *   DIT_BLOCK_ADALN: ada.w [4d, d], ada.b [4d] with rows (shift1, scale1, shift2, scale2);
 *   DIT_BLOCK_IN_CONTEXT: ln1.g [d], ln1.b [d] replace ada.w, ada.b, and ln2.g [d], ln2.b [d]
 *       come before fc1.w; DIT_BLOCK_CROSS_ATTN: the same, plus after proj.b: xln.g [d],
 *       xln.b [d], xq.w [d, d], xq.b [d], xkv.w [2d, d] (rows [k | v]), xkv.b [2d], xo.w [d, d],
 *       xo.b [d]; for both, final.ln.g [d], final.ln.b [d] replace final.ada.w, final.ada.b.
 * The library copies everything; the caller may free the host arrays on return.
 * Blocks the calling thread until the upload is complete.
 * Returns DIT_ERR_INVALID_ARG / DIT_ERR_UNSUPPORTED before any CUDA call when the
 * configuration is rejected, DIT_ERR_NO_DEVICE without an sm_100 device, DIT_ERR_OOM
 * when device memory runs out.  *out is set only on DIT_OK.
 */
dit_status dit_create(const dit_config* cfg, const float* const* weights, int n_weights,
                      dit_handle** out);

/* Number of weight arrays dit_create expects for cfg (0 if cfg is invalid). */
int dit_weight_count(const dit_config* cfg);

/*
 * dit_forward — one denoiser evaluation, enqueued on stream.
 *   x   dev float32 [B, C, H, W] (images) or [B, C, F, H, W] (video), NC(F)HW
 *   t   dev float32 [B] timesteps
 *   y   dev int32 [B] class labels (DIT_COND_CLASS) or float32 [B, d] (DIT_COND_VECTOR)
 *   out dev float32 [B, C_out, (F,) H, W]
 * Guidance: with a class-conditional model and cfg_scale != 1 the library runs 2B
 * rows, [x; x] with labels [y; num_classes], and writes e(null) + s (e(y) - e(null))
 * on every output channel (or on the first n only, see DIT_OPT_CFG_CHANNELS).
 * Otherwise it runs B rows and writes e(y).  1 <= B <= max_batch.
 * One forward may be in flight per handle (the handle owns one workspace); the
 * handle is not thread-safe.  Buffers must stay valid until the stream reaches
 * the end of the call.
 */
dit_status dit_forward(dit_handle* h, const float* x, const float* t, const void* y, int B,
                       float cfg_scale, float* out, dit_stream_t stream);

/*
 * dit_forward_host — dit_forward on host buffers: copies x, t, y into the handle's
 * device staging area, runs the forward on stream, copies out back and waits for
 * the stream.  Same layouts and rules as dit_forward.
 */
dit_status dit_forward_host(dit_handle* h, const float* x_host, const float* t_host,
                            const void* y_host, int B, float cfg_scale, float* out_host,
                            dit_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* Sampling: the update around the denoiser.                                      */
/* ------------------------------------------------------------------------------ */

enum { DIT_SAMPLER_DDIM = 0, DIT_SAMPLER_EULER = 1 };

/*
 * dit_sampler_step — one sampler update of the latent x given the denoiser output
 * model_out of dit_forward (one fused elementwise kernel):
 *   DIT_SAMPLER_DDIM  (noise head): eps = the first C of the C_out output channels (a
 *       learned-covariance head writes [eps | Sigma]); with a = abar now, b = abar next,
 *       x_next = sqrt(b) (x - sqrt(1-a) eps) / sqrt(a) + sqrt(1-b) eps, i.e. the clean
 *       latent that eps implies under the DDPM forward process x_t = sqrt(abar_t) x_0 +
 *       sqrt(1-abar_t) eps ("Sora / DiT", method section, training-objective bullet)
 *       carried to level b with the same eps.  The two coefficients are formed on the host
 *       in double precision.
 *   DIT_SAMPLER_EULER (velocity head): x_next = x + (b - a) v, v = the first C channels,
 *       with a = t now, b = t next, one Euler step along x_t = t x_1 + (1-t) x_0 ("GOKU",
 *       §2.3 rectified flow).
 * x, x_next: device float32 [B, C, F, H, W] (F omitted for images); x_next may equal x.
 * model_out: device float32 [B, C_out, F, H, W].  Asynchronous on `stream`.
 * Errors (nothing is launched): DIT_ERR_INVALID_ARG for null pointers, B outside
 * [1, max_batch], an unknown kind, or DDIM levels outside (0, 1].
 */
dit_status dit_sampler_step(dit_handle* h, int kind, const float* x, const float* model_out, int B, float a,
                            float b, float* x_next, dit_stream_t stream);

/*
 * dit_sample — `steps` sampling steps in place on x: for i = 0 .. steps-1,
 *   out = dit_forward(x, t = model_t[i] for every sample, y, B, cfg_scale) into the
 *         handle's own output buffer, then
 *   x   = dit_sampler_step(kind, x, out, levels[i], levels[i+1]).
 * x: device float32 [B, C, F, H, W] (in: the starting noise; out: the sample).
 * y: device labels / text vectors as for dit_forward.  model_t: host float[steps], the
 * timestep value the denoiser sees at step i; levels: host float[steps+1] (abar for DDIM,
 * t for Euler).  Both host arrays are read before the call returns; the work is
 * asynchronous on `stream`.  With DIT_OPT_USE_GRAPH the whole loop (steps forwards and
 * updates) is captured and replayed like dit_forward: a call that repeats the previous
 * call's pointers, batch, cfg_scale, kind and levels replays the graph (model_t is
 * uploaded every call, so it may change).  Errors as dit_forward and dit_sampler_step,
 * plus DIT_ERR_INVALID_ARG for steps < 1 or null host arrays; nothing is launched then.
 */
dit_status dit_sample(dit_handle* h, int kind, float* x, const void* y, int B, float cfg_scale, int steps,
                      const float* model_t, const float* levels, dit_stream_t stream);

/* Reads and clears the handle's device status word (synchronises the device first).
   Returns DIT_OK or the first device-side error recorded since the last call. */
dit_status dit_sync_status(dit_handle* h);

/* Text of the last host-side error on this handle (never NULL). */
const char* dit_last_error(const dit_handle* h);

/* Short name of a status code (never NULL). */
const char* dit_status_string(dit_status s);

/* Frees every device allocation of the handle.  Waits for outstanding work. */
void dit_destroy(dit_handle* h);

/* ------------------------------------------------------------------------------ */
/* Diagnostics.  Same device-pointer and stream rules as dit_forward.             */
/* ------------------------------------------------------------------------------ */

/* Option switches (test use).  DIT_OPT_FORCE_GUIDANCE = 1 makes dit_forward run the
   2B guided rows even at cfg_scale == 1 (so e(null) + 1*(e(y)-e(null)) is returned).
   DIT_OPT_USE_GRAPH = 0/1 (default 0) disables / enables CUDA-graph replay of the forward:
   for dit_forward and dit_forward_host, a call whose device pointers, batch and cfg_scale
   repeat the previous call's runs directly the first time, is captured into a graph (on a
   private stream) the second time and then replays as one graph launch on the caller's
   stream.  New pointers or parameters start over; the contents of the buffers may change
   freely.  While profiling is enabled the graph is bypassed.  If the capture fails the
   option turns itself off and the call runs directly.
   DIT_OPT_OVERLAP_LAUNCH = 0/1 (process-wide, default 1): launch each kernel with
   programmatic dependent launch so its set-up overlaps the tail of the previous one.
   DIT_OPT_CFG_CHANNELS = n >= 0 (default 0 = every channel): classifier-free guidance
   combines only output channels c < n; the other channels return the conditional
   prediction.  n = 3 is the variant that "확산 트랜스포머" ("ImageNet 클래스 조건 생성")
   attributes to the official code; guidance on every channel is the standard form.
   A negative n is DIT_ERR_INVALID_ARG.
   DIT_OPT_REPEAT_KIND = k (a DIT_KERNEL_* kind, default -1 = off): a timing diagnostic that
   launches every kernel of kind k twice where the forward launches it once, so that the step
   time grows by that kind's in-pipeline cost (the second launch repeats the same work on the
   same buffers; for the residual kinds DIT_KERNEL_PROJ and DIT_KERNEL_FC2 it adds the update
   twice, so outputs are meaningless while it is on).  Part of the graph cache key.
   DIT_OPT_SPLIT_K = s (1..8, default 1): the residual GEMMs with a short reduction (the
   d-wide out-projections) split K into s slices, each adding its share into the residual
   stream.  The slices' additions reach memory in no fixed order, so with s > 1 repeated
   forwards may differ in float32 rounding (not bit-identical); s = 1 is deterministic.
   DIT_OPT_PAIR_GEMM = 0/1 (default 0): run the bf16 block GEMMs (QKV without QK norm / RoPE,
   out-projection, FFN) on SM pairs, tcgen05.mma.cta_group::2 with 256 x 256 tiles: each SM
   loads its 128 rows of A and half of B per stage (32 KB instead of 48 KB), so six stages fit
   instead of four.  The split-K option does not apply to the pair kernels. */
enum { DIT_OPT_FORCE_GUIDANCE = 1, DIT_OPT_USE_GRAPH = 2, DIT_OPT_OVERLAP_LAUNCH = 3, DIT_OPT_CFG_CHANNELS = 4,
       DIT_OPT_REPEAT_KIND = 5, DIT_OPT_SPLIT_K = 6, DIT_OPT_PAIR_GEMM = 7 };
dit_status dit_set_option(dit_handle* h, int option, int value);

/*
 * dit_debug_residual — run the forward up to and including block `after_block`
 * (0 = right after patch embedding) and copy the float32 residual stream
 * [rows, T, d] into h_out (dev), rows ordered [cond; uncond] when guided.
 * The final layer is not run.  Same guidance rule as dit_forward.
 */
dit_status dit_debug_residual(dit_handle* h, const float* x, const float* t, const void* y, int B,
                              float cfg_scale, int after_block, float* h_out, dit_stream_t stream);

/*
 * dit_debug_condition — compute the condition vector c [rows, d] (float32, dev)
 * from t and y exactly as dit_forward does (rows = 2B when guided).
 */
dit_status dit_debug_condition(dit_handle* h, const float* t, const void* y, int B, float cfg_scale,
                               float* c_out, dit_stream_t stream);

/*
 * dit_debug_wait_probe — launch one kernel that waits on a device flag nothing ever
 * sets, with the library's bounded-wait routine and a limit of timeout_us
 * microseconds.  When the limit runs out the kernel records DIT_ERR_DEVICE_TIMEOUT
 * in the status word and returns, so dit_sync_status reports it and the context
 * stays usable.  Exercises the device-side failure path without faulting a GPU.
 */
dit_status dit_debug_wait_probe(dit_handle* h, int timeout_us, dit_stream_t stream);

/*
 * dit_op_linear_bf16 — the tensor-core GEMM building block on its own:
 *   y[M, N] = x[M, K] W[N, K]^T + b[N]
 * x, W: dev bf16 (raw uint16 bit patterns), row-major, K % 8 == 0, 16-byte aligned;
 * b: dev float32 [N] or NULL; y: dev float32 [M, N].  block_n selects the tile
 * width (16, 32, 64, 128, 144 or 256).  Uses tcgen05.mma with TMA-fed shared
 * memory and a TMEM accumulator; float32 accumulation.
 */
dit_status dit_op_linear_bf16(const uint16_t* x, const uint16_t* w, const float* b, float* y,
                              int M, int N, int K, int block_n, dit_stream_t stream);

/*
 * Per-step kernel timing.  While enabled, dit_forward brackets launches with a pair of CUDA
 * events on its stream and files the pair under one of the DIT_KERNEL_* kinds: every launch
 * (enable = 1) or only the launches of kind k (enable = 2 + k), so that the other kernels
 * keep their programmatic-dependent-launch overlap.  The graph is bypassed while profiling.
 * dit_profile_read synchronises the device, writes per-kind total milliseconds and
 * launch counts (arrays of at least DIT_KERNEL_COUNT entries) and clears the record.
 */
enum { DIT_KERNEL_COND = 0, DIT_KERNEL_ADALN = 1, DIT_KERNEL_PATCH = 2, DIT_KERNEL_LN = 3, DIT_KERNEL_QKV = 4,
       DIT_KERNEL_ATTN = 5, DIT_KERNEL_PROJ = 6, DIT_KERNEL_FC1 = 7, DIT_KERNEL_FC2 = 8, DIT_KERNEL_DECODE = 9,
       DIT_KERNEL_SAMPLER = 10, DIT_KERNEL_COUNT = 11 };
dit_status dit_profile_enable(dit_handle* h, int enable);
dit_status dit_profile_read(dit_handle* h, float* total_ms, int* launches);

/*
 * dit_condition_static — the condition vector c [rows, hidden] (rows = 2B when
 * guided, else B), computed like dit_forward computes it, for callers that cannot
 * allocate device memory (code that runs where cudaMalloc is forbidden or would
 * deadlock, such as inside a caching allocator's own callbacks, or programs that
 * must fix their whole device footprint before they start).  No handle is needed and
 * nothing is allocated: every input, weight and output is the caller's, and the
 * intermediate buffers live in one fixed device array inside the library.
 * The pages have no counterpart of this entry point; it is a library service.
 *   t [B] f32, y int32 [B] (cond_kind DIT_COND_CLASS) or f32 [B, hidden] (DIT_COND_VECTOR),
 *   w1 [hidden, freq_dim], b1 [hidden], w2 [hidden, hidden], b2 [hidden],
 *   table [num_classes+1, hidden] (class models; NULL otherwise), all dev float32;
 *   guided = 1 appends B rows with the null label (class models only);
 *   c_out dev f32 [rows, hidden]; status dev int32 (or NULL) receives DIT_ERR_BAD_LABEL
 *   when a label lies outside [0, num_classes] (the label is clamped).
 * Limits of the fixed scratch: rows <= 128, freq_dim <= 512, hidden <= 1536 (both multiples
 * of 4); other requests return DIT_ERR_INVALID_ARG before anything is launched.  The array
 * (1.75 MiB) stays resident on every GPU that loaded the library until the process
 * exits.  The first call on a device looks up the array's device address (once per
 * device, with that device current; again after a device reset gives the device a new
 * context); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents; every call
 * rewrites what it reads, so nothing has to start at zero, but calls whose work
 * overlaps on the GPU (different streams, or different threads) race on it.
 */
dit_status dit_condition_static(const float* t, const void* y, int B, int guided, const float* w1,
                                const float* b1, const float* w2, const float* b2, const float* table,
                                int cond_kind, int num_classes, int freq_dim, int hidden, float t_scale,
                                float* c_out, int* status, dit_stream_t stream);

/*
 * dit_op_linear_bf16_pair — the same product on SM pairs: a cluster of two CTAs
 * issues tcgen05.mma.cta_group::2 on 256 x block_n output tiles, each SM loading half
 * of the A rows and half of the W rows of every stage.  block_n: 64, 128, 144, 192 or
 * 256.  Same argument rules as dit_op_linear_bf16.
 */
dit_status dit_op_linear_bf16_pair(const uint16_t* x, const uint16_t* w, const float* b, float* y,
                                   int M, int N, int K, int block_n, dit_stream_t stream);

/*
 * dit_op_linear_e4m3 — the FP8 tensor-core GEMM building block (tcgen05.mma kind::f8f6f4):
 *   y[m, n] = sx[m] sw[n] sum_k x[m, k] w[n, k] + b[n]
 * x [M, K], w [N, K]: dev FP8 E4M3 bytes, row-major, K % 16 == 0, 16-byte aligned;
 * sx [M], sw [N]: dev float32 scales; b: dev float32 [N] or NULL; y: dev float32 [M, N].
 * block_n: 64, 128 or 256.  float32 accumulation.  Asynchronous on `stream`.
 */
dit_status dit_op_linear_e4m3(const uint8_t* x, const uint8_t* w, const float* sx, const float* sw, const float* b,
                              float* y, int M, int N, int K, int block_n, dit_stream_t stream);

/*
 * dit_op_attention_bf16 — the tensor-core attention kernel of the bf16 forward on its own:
 *   o[r, tau, h*dh : (h+1)*dh] = softmax(q_{r,h} k_{r,h}^T / sqrt(dh)) v_{r,h}   (full, no mask)
 * for every sample row r < R and head h < H ("확산 트랜스포머", section "adaLN-Zero": Attn is
 * multi-head self-attention over all T tokens).  Layouts (dev bf16 bit patterns, the forward's
 * own workspace layouts; Tpad = T rounded up to a multiple of 128, DP = dh rounded up to a
 * multiple of 16):
 *   q, k [R*H, Tpad, DP]  row-major, rows >= T and columns >= dh must hold zeros;
 *   v    [R*H, DP, Tpad]  V transposed, same zero padding;
 *   o    [R*T, H*dh]      token-major output.
 * dh must be 64 or 72 (DIT_ERR_UNSUPPORTED otherwise).  counters: dev int32[2] or NULL;
 * counters[0] receives DIT_ERR_DEVICE_TIMEOUT if a bounded wait runs out, and counters[1] is
 * incremented once per warp of 32 query rows each time the online softmax moves its
 * reference maximum (and rescales its running output) because the row maximum grew by more
 * than 2^8 — a diagnostic of that code path.  Asynchronous on `stream`.
 */
dit_status dit_op_attention_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int R, int H,
                                 int T, int dh, int* counters, dit_stream_t stream);

/* Reads and clears the handle's count of attention reference-maximum moves (the same event
   as counters[1] of dit_op_attention_bf16), accumulated over every bf16 forward since the
   last read.  Synchronises the device first. */
dit_status dit_debug_attention_rescales(dit_handle* h, long long* count);

/* Number of kernel launches one dit_forward enqueues for batch B (graph nodes if a
   graph is replayed). */
int dit_forward_launch_count(const dit_handle* h, int B, float cfg_scale);

#ifdef __cplusplus
}
#endif

#endif /* DIT_B200_H */
