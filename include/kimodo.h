/*
 * kimodo.h -- C ABI of the B200 (sm_100a) two-stage DDIM motion denoiser.
 *
 * The library runs the denoising loop of a Kimodo-style text-to-motion model on
 * one GPU: per DDIM step a root transformer, the global-to-local root transform,
 * a body transformer, classifier-free guidance and the DDIM x(t-1) update
 * ("Kimodo WebGPU" page, "Architecture" figure and "Model details" table).
 * The text encoder is not part of the library: 4096-float embeddings are inputs.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Return value: KIMODO_OK (0) or a negative KIMODO_E* status; the message of the
 *   last failure on the calling thread is available from kimodo_last_error().
 *   No exception or abort crosses this boundary.
 * Pointers: every tensor argument may be HOST memory (pageable or pinned) or
 *   DEVICE memory of the context's GPU; the library detects which.  Host inputs
 *   are copied to device staging on `stream`; when any output is host memory the
 *   call synchronises `stream` before returning, otherwise it returns once the
 *   work is enqueued (asynchronous).  The caller keeps ownership of all tensors.
 * Layouts: row-major float32, C order.  Motion features per frame are
 *   [root 5 | body 274] = 279 floats; root 5 = (x, z, sin heading,
 *   cos heading, height); body 274 = 30 joints x (3 position + 6D rotation) +
 *   4 foot contacts.
 * Masking: frames at index >= lengths[b] are padding.  Their input values,
 *   whatever they are (NaN included), never reach a valid output, and every
 *   output writes 0 there.
 * stream: a cudaStream_t cast to void*; NULL means the legacy default stream.
 * Device-side failures (a bounded wait in a kernel that ran out) are reported
 *   by kimodo_sync_status() and by the next call on the context.
 */
#ifndef KIMODO_H
#define KIMODO_H

#include <stddef.h>

#if defined(__GNUC__)
#define KIMODO_API __attribute__((visibility("default")))
#else
#define KIMODO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kimodo_ctx kimodo_ctx;

enum {
  KIMODO_OK = 0,
  KIMODO_EINVAL = -1,       /* bad argument (message says which) */
  KIMODO_ENOMEM = -2,       /* device or host allocation failed */
  KIMODO_ECUDA = -3,        /* a CUDA runtime/driver call failed */
  KIMODO_EUNSUPPORTED = -4, /* no sm_100 device, or the kernels are missing */
  KIMODO_ETIMEOUT = -5      /* a kernel's bounded wait gave up */
};

enum { KIMODO_FP32 = 0, KIMODO_BF16 = 1 };
enum { KIMODO_NET_ROOT = 0, KIMODO_NET_BODY = 1 };

/* Model constants ("Kimodo WebGPU", "Model details": 16-layer post-norm encoders,
 * 1024 hidden, 8 heads x 128, 2048 FFN; 282M parameters in all). */
#define KIMODO_N_PARAMS 281963799u
#define KIMODO_TEXT_DIM 4096
#define KIMODO_MOTION_DIM 279
#define KIMODO_ROOT_DIM 5
#define KIMODO_BODY_DIM 274
#define KIMODO_MAX_FRAMES 300

/*
 * Create a context on CUDA device `device` and upload the weights.
 *
 * host_blob: n_floats float32 values in the canonical order (root network, then
 *   body network; per network: text projection W[1024x4096], b[1024]; timestep
 *   MLP W1[1024x1024], b1, W2[1024x1024], b2; input projection W[1024xDin], b;
 *   16 x (qkv W[3072x1024] with rows Q,K,V, qkv b[3072], out-proj W[1024x1024],
 *   b, LayerNorm-1 gamma, beta, FFN-1 W[2048x1024], b[2048], FFN-2 W[1024x2048],
 *   b, LayerNorm-2 gamma, beta); output projection W[Doutx1024], b[Dout]).
 *   Din/Dout = 5/5 (root) and 279/274 (body).  Matrices are [out x in].
 *   Read during the call only; host or device memory.
 * n_floats: must equal KIMODO_N_PARAMS, else KIMODO_EINVAL.
 * precision: KIMODO_BF16 (tensor-core path: bf16 operands, fp32 accumulation,
 *   fp32 LayerNorm/softmax/DDIM) or KIMODO_FP32 (fp32 everywhere).
 * On success *ctx receives a context owned by the caller (kimodo_free).
 */
KIMODO_API int kimodo_load_weights(kimodo_ctx** ctx, const float* host_blob, size_t n_floats,
                        int precision, int device);

/*
 * One sub-network forward ("Kimodo WebGPU", "Model details": one 16-layer
 * TransformerEncoder).  Sequence = [condition token | T frame tokens]; the
 * condition token is TextProj(emb) + TimestepMLP(sinusoid(t)).
 *
 * net: KIMODO_NET_ROOT (Din=5, Dout=5) or KIMODO_NET_BODY (Din=279, Dout=274).
 * x: [batch, frames, Din] input features.  emb: [batch, 4096] text embeddings.
 * t: diffusion timestep in [0, 999].  lengths: int32 [batch], 1..frames.
 * out: [batch, frames, Dout] network output (padded frames written as 0).
 * 1 <= batch, 1 <= frames <= 300.
 */
KIMODO_API int kimodo_denoiser_forward(kimodo_ctx* ctx, int net, const float* x, const float* emb, int t,
                            const int* lengths, int batch, int frames, float* out, void* stream);

/*
 * Allocation-free variant of kimodo_denoiser_forward (the pages describe no
 * counterpart: it serves callers of this library that must not allocate device
 * memory).  Some callers cannot call cudaMalloc: an engine or runtime that owns
 * every byte of device memory through its own allocator or a fixed budget, and
 * latency-sensitive callers that cannot afford the device-wide synchronisation a
 * cudaMalloc or cudaFree may cause.  kimodo_denoiser_forward allocates its
 * activation workspace on first use; this call instead uses a static device array
 * of the library (about 19 MiB, held by every GPU that loads the library until
 * the process exits) and calls no cudaMalloc, cudaFree or other allocating
 * routine.  The context itself is created, with its weights, by
 * kimodo_load_weights.
 *
 * Arguments and output layout are those of kimodo_denoiser_forward, within these
 * limits: batch <= 16 and batch * (frames + 1) <= 512 tokens, else KIMODO_EINVAL
 * (use kimodo_denoiser_forward for larger calls).  The scratch always holds the
 * padded token layout (every sequence frames + 1 rows, padded rows computed and
 * discarded), where kimodo_denoiser_forward packs the valid tokens when host lengths
 * are shorter than frames; the results agree within the path's tolerances (bf16:
 * relative L2 2e-2; fp32: max-abs relative 1e-4), not necessarily bit for bit.
 * The first call on a device looks up the array's device address (set-up, cached per
 * device for the life of the process; a cudaDeviceReset invalidates it together with
 * every context); make that first call before any stream capture.  Every call on a
 * device shares the one array and overwrites the previous call's contents: calls
 * whose work can overlap on the GPU (other streams, other contexts, other threads)
 * race and must be ordered by the caller.
 */
KIMODO_API int kimodo_denoiser_forward_noalloc(kimodo_ctx* ctx, int net, const float* x, const float* emb,
                                               int t, const int* lengths, int batch, int frames,
                                               float* out, void* stream);

/*
 * One two-stage DDIM step with classifier-free guidance, cond and uncond
 * batched in one pass per network:
 *   per branch: root = Root(x_t[..., :5]); local = G2L(root);
 *               body = Body([x_t[..., 5:] | local]); x0_branch = [root | body]
 *   x0 = x0_u + cfg_scale (x0_c - x0_u)
 *   x_prev = sqrt(ab_prev) x0 + sqrt(1 - ab_prev) (x_t - sqrt(ab_t) x0) / sqrt(1 - ab_t)
 * with ab the linear-beta (1e-4..0.02, 1000 steps) cumulative product, ab(-1) = 1.
 *
 * x_t: [batch, frames, 279].  text_emb: [batch, 4096].  null_emb: [4096]
 *   (broadcast) or [batch, 4096], pass null_batch = 1 or batch.
 * t in [0, 999], t_prev in [-1, t).  cfg_scale finite.
 * x_prev: [batch, frames, 279]; may alias x_t.
 */
KIMODO_API int kimodo_ddim_step(kimodo_ctx* ctx, const float* x_t, const float* text_emb,
                     const float* null_emb, int null_batch, const int* lengths, int batch,
                     int frames, int t, int t_prev, float cfg_scale, float* x_prev, void* stream);

/*
 * Full DDIM sampling loop: `steps` two-stage steps (as kimodo_ddim_step) on the
 * trailing timesteps t_k = floor(1000 (steps - k) / steps + 1/2) - 1, k = 0..steps-1,
 * t_prev = t_{k+1}, and -1 after the last step (for steps dividing 1000 this is
 * t_k = 999 - k (1000/steps)), starting from `noise`; 1 <= steps <= 1000.  The loop
 * runs as one CUDA graph captured per (batch, frames, steps, cfg_scale, sampler
 * options) and cached in the context; no host synchronisation happens between steps.
 *
 * noise: [batch, frames, 279].  out: [batch, frames, 279] final sample; may alias noise.
 */
KIMODO_API int kimodo_ddim_sample(kimodo_ctx* ctx, const float* text_emb, const float* null_emb,
                       int null_batch, const float* noise, const int* lengths, int batch,
                       int frames, int steps, float cfg_scale, float* out, void* stream);

/*
 * Sampler options of the _ex entry points (the "Model details" table of the
 * "Kimodo WebGPU" page names a cosine beta schedule; the DDIM paper, Song, Meng &
 * Ermon 2021, eqs. 12 and 16, defines the eta > 0 family).
 *
 * schedule: KIMODO_SCHEDULE_LINEAR (beta = linspace(1e-4, 0.02, 1000), the default)
 *   or KIMODO_SCHEDULE_COSINE (Nichol & Dhariwal 2021: alphabar(u) = f(u) / f(0),
 *   f(u) = cos^2((u + 0.008) / 1.008 * pi / 2), beta_i = min(1 - alphabar((i+1)/1000) /
 *   alphabar(i/1000), 0.999), table = cumulative product of 1 - beta).
 * eta: in [0, 1].  With sigma = eta sqrt((1 - ab_prev) / (1 - ab_t)) sqrt(1 - ab_t / ab_prev):
 *   x_prev = sqrt(ab_prev) x0 + sqrt(1 - ab_prev - sigma^2) eps + sigma z,
 *   eps = (x_t - sqrt(ab_t) x0) / sqrt(1 - ab_t); eta = 0 is deterministic DDIM.
 * step_noise: the standard-normal draws z (fp32, host or device memory, read during
 *   the call's work; the caller keeps it alive until then): [steps, batch, frames, 279]
 *   for kimodo_ddim_sample_ex (step k uses slice k), [batch, frames, 279] for
 *   kimodo_ddim_step_ex.  Required when eta > 0, ignored when eta = 0.  Values at
 *   padded frames are never read into valid outputs.  A graph captured for a device
 *   step_noise pointer reads that pointer on every replay.
 * text_batch: 0 (text_emb has `batch` rows), or a divisor of batch for variations of
 *   fewer prompts: text_emb then has text_batch rows and sequence b uses row
 *   b / (batch / text_batch), each take with its own noise rows (the pages generate
 *   several takes of one prompt in a batch).  null_emb keeps its own broadcast rule.
 * A NULL options pointer means { KIMODO_SCHEDULE_LINEAR, 0, NULL, 0 }.
 */
enum { KIMODO_SCHEDULE_LINEAR = 0, KIMODO_SCHEDULE_COSINE = 1 };
typedef struct kimodo_sampler {
  int schedule;
  float eta;
  const float* step_noise;
  int text_batch;
} kimodo_sampler;

/* kimodo_ddim_sample with sampler options (KIMODO_EINVAL on an unknown schedule,
 * eta outside [0, 1] or not finite, eta > 0 without step_noise, or a text_batch that
 * does not divide batch). */
KIMODO_API int kimodo_ddim_sample_ex(kimodo_ctx* ctx, const float* text_emb, const float* null_emb,
                       int null_batch, const float* noise, const int* lengths, int batch,
                       int frames, int steps, float cfg_scale, const kimodo_sampler* options,
                       float* out, void* stream);

/* kimodo_ddim_step with sampler options (same checks as kimodo_ddim_sample_ex). */
KIMODO_API int kimodo_ddim_step_ex(kimodo_ctx* ctx, const float* x_t, const float* text_emb,
                     const float* null_emb, int null_batch, const int* lengths, int batch,
                     int frames, int t, int t_prev, float cfg_scale, const kimodo_sampler* options,
                     float* x_prev, void* stream);

/* Synchronise `stream` and report any device-side failure recorded since the
 * last check (KIMODO_ETIMEOUT with the kernel named in kimodo_last_error()). */
KIMODO_API int kimodo_sync_status(kimodo_ctx* ctx, void* stream);

/* Diagnostic of the device error path: enqueue on `stream` one kernel whose bounded
 * wait, on a barrier that nothing completes, gives up after limit_us microseconds
 * (1 .. 2000000) and records KIMODO_ETIMEOUT in the context's error word, as the path's
 * kernels do when one of their waits runs out.  No fault and no unbounded wait occur;
 * kimodo_sync_status() then reports the timeout ("wait self-test") and clears it, and
 * the context stays usable.  While the error is recorded, the tensor-core kernels of
 * calls enqueued after it skip their work. */
KIMODO_API int kimodo_wait_selftest(kimodo_ctx* ctx, int limit_us, void* stream);

/* Per-kernel-class timing of the next calls (instrumentation, off by default).
 * With enable != 0, every launch is bracketed by CUDA events; kimodo_ddim_sample
 * then captures a fresh, uncached graph whose kernel nodes sit between timing
 * event nodes (so the times carry no host gaps, but consecutive kernels no longer
 * overlap through programmatic dependent launch), runs it and waits for it.
 * kimodo_profile_read() returns, for each of
 * n_classes <= 8 classes (0 tensor-core GEMM, 1 attention, 2 LayerNorm,
 * 3 elementwise/motion, 4 fp32 GEMM, 5 setup), the summed milliseconds, the
 * number of launches and the algorithmic FLOPs and bytes since the last reset. */
KIMODO_API int kimodo_profile_enable(kimodo_ctx* ctx, int enable);
KIMODO_API int kimodo_profile_read(kimodo_ctx* ctx, int n_classes, double* ms, long long* launches,
                        double* flops, double* bytes);

/* Number of this library's kernel launches enqueued by the last completed
 * sample/step/forward call (graph nodes included). */
KIMODO_API long long kimodo_last_launch_count(kimodo_ctx* ctx);

/* Release the context and all device memory it owns.  NULL is accepted. */
KIMODO_API void kimodo_free(kimodo_ctx* ctx);

/* Message of the last failure on the calling thread ("" if none). */
KIMODO_API const char* kimodo_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KIMODO_H */
