/*
 * libgdn: the frame-wise Gated DeltaNet (GDN) scan on NVIDIA B200 (sm_100a).
 *
 * The operation ("NVIDIA Apresenta SANA-WM: Um Modelo de Mundo de Larga
 * Escala ...", acheiumaia.com.br, section "A Arquitetura: Quatro Decisoes de
 * Design Centrais", item "1. Atencao Linear Hibrida com Gated DeltaNet"):
 * every latent frame of S spatial tokens is one recurrent step on a constant
 * D x D state per head, with a decay gate gamma, a delta-rule correction and
 * keys scaled by 1/sqrt(D*S). Per head and frame t, with K_t, Q_t, V_t of
 * shape S x D, s = 1/sqrt(D*S) and M of shape D x D:
 *
 *     W   = (s K_t) M_{t-1}
 *     R   = V_t - gamma_t W
 *     M_t = gamma_t M_{t-1} + beta_t (s K_t)^T R
 *     O_t = Q_t M_t
 *
 * Layouts (all row-major, contiguous, element strides implied by the sizes):
 *   q, k, v, out   [B][H][T][S][D]   scan;  [B][H][S][D] step (T = 1)
 *   gamma, beta    [B][H][T] float   scan;  [B][H] float      step
 *   state_in/out   [B][H][D][D] float; element [i][j]: i = key dim, j = value dim
 * Keys are passed unscaled: the library applies s = 1/sqrt(D*S) itself.
 * Gates are used as given (not clamped or validated; NaN propagates).
 *
 * Pointers: every array pointer is a DEVICE pointer of the current CUDA
 * device. The caller owns every buffer; the library keeps no pointer after a
 * call returns. Device memory: a bf16 scan that runs the tensor-core kernel
 * with more than one CTA per head (see gdn_plan) takes stream-ordered scratch
 * for the transition operands the CTAs of a head share (16 frames x 24 KiB
 * per head, plus 8 bytes x (16 + CTAs per head) of flags), with
 * cudaMallocAsync on `stream`, and releases it with cudaFreeAsync on the same
 * stream right after the launch; every other call allocates no device
 * memory. q, k, v, out, state_in and
 * state_out must be 16-byte aligned; gamma and beta 4-byte aligned.
 * state_in == NULL means M_0 = 0. state_out == NULL means the final state is
 * not written. state_in may equal state_out (the update is then in place);
 * out must not overlap q, k, v or the states.
 *
 * Ordering: work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 * default stream) and the call returns without waiting for it. Arguments
 * are checked first, on the host; on any error nothing is enqueued and a
 * negative gdn_status is returned.
 *
 * Device-side waits inside the kernels are bounded. A kernel whose wait runs
 * out stops early, leaves its outputs incomplete and records
 * GDN_ERR_TIMEOUT in a device status word; read it with gdn_device_status().
 */
#ifndef LIBGDN_GDN_H_
#define LIBGDN_GDN_H_

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_VERSION_MAJOR 1
#define GDN_VERSION_MINOR 0
#define GDN_VERSION_PATCH 0

typedef enum gdn_status {
  GDN_OK = 0,
  GDN_ERR_NULL = -1,            /* q, k, v, gamma, beta or out is NULL */
  GDN_ERR_SHAPE = -2,           /* B, H, T or S < 1, or a size overflows 64 bits */
  GDN_ERR_UNSUPPORTED_D = -3,   /* D not in {32, 64, 128} */
  GDN_ERR_ALIGN = -4,           /* a pointer breaks the alignment rules above */
  GDN_ERR_CUDA = -5,            /* a CUDA runtime or driver call failed */
  GDN_ERR_TIMEOUT = -6,         /* a device-side wait ran out (from gdn_device_status) */
  GDN_ERR_ALIAS = -7,           /* out overlaps an input or a state buffer */
  GDN_ERR_SCRATCH = -8,         /* gdn_frame_scan_noalloc: a ring plan with B * H > GDN_NOALLOC_MAX_HEADS */
  GDN_ERR_FLAGS = -9,           /* unknown bits in `flags` (the _ex calls) */
  GDN_ERR_UNSUPPORTED = -10     /* gdn_frame_step_rope, gdn_frame_stream(_rope): sizes their kernel does not take */
} gdn_status;

/* bf16 scan over T frames. q, k, v, out hold bf16 bit patterns (uint16).
 * Arithmetic (D = 64 and 128, tensor-core kernels): K^T K and K^T V
 * accumulate in fp32 on tcgen05 tensor cores; the state M is kept in fp32 on
 * chip across all T frames and updated as M <- gamma M + A' M + c in fp32,
 * where the product A' M (A' = -gamma beta s^2 K^T K; at D = 128 it is
 * accumulated onto K^T V before the scale beta s) and the read-out Q M take M
 * and A' rounded to bf16 with fp32 accumulation; out is rounded to bf16
 * (round to nearest even). D = 64 runs a cluster of 1, 2 or 4 CTAs per head
 * (gdn_plan); D = 128 a cluster of two, one streaming K and V and running the
 * recurrence, one streaming Q and writing out. A single frame at D = 64 runs
 * the row-split kernel of gdn_frame_step. D = 32 runs the update in fp32 on
 * CUDA cores.
 * On the seeded rollout workload the per-frame relative error against a
 * float64 reference is about 2.4e-3 for out and 2e-6 for the final state. */
GDN_API int gdn_frame_scan(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int T, int S, int D, void* stream);

/* One bf16 frame (T = 1) for chunk-causal rollout: the state is read from
 * state_in and written to state_out, which may be the same buffer, so a
 * caller can carry it across calls. This is the sequential rollout variant
 * the SANA-WM article names among its three inference modes ("NVIDIA
 * Apresenta SANA-WM ...", acheiumaia.com.br, the paragraph on the
 * bidirectional, chunk-causal autoregressive and distilled generators): one
 * latent frame arrives per call and the constant-size D x D state carries the
 * whole history. Same update and precision as gdn_frame_scan (the
 * state-dependent product takes A' and M in bf16); a chain of steps matches
 * one scan over the same frames to fp32 rounding. */
GDN_API int gdn_frame_step(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int S, int D, void* stream);

/* gdn_frame_scan for callers that must not allocate device memory. The
 * method has no counterpart to this entry point: it exists for the library's
 * users, not for the operation.
 *
 * Who needs it: a caller that has reserved nearly all of the GPU's memory for
 * its own pool up front (an inference engine, say) cannot let a library take
 * more during a call, since the allocation would fail or push out its cache;
 * a process with a hard device-memory cap is in the same place; and a caller
 * in a tight loop may not accept the cost of an allocation at all (cudaMalloc
 * and cudaFree can synchronize the device, and a stream-ordered pool may have
 * to grow). gdn_frame_scan takes stream-ordered scratch when it runs with
 * more than one CTA per head; this entry point takes that scratch from one
 * fixed array in the library's device code instead, and calls no cudaMalloc,
 * cudaMallocAsync, cudaFree or cudaFreeAsync.
 *
 * Limit: the scratch is the transition-operand ring, which only a plan with
 * the tensor-core kernel and more than one CTA per head uses (gdn_plan). For
 * such a plan B * H must be <= GDN_NOALLOC_MAX_HEADS (32); a larger one
 * returns GDN_ERR_SCRATCH, after the argument checks every entry point makes,
 * and enqueues nothing. Other plans take no scratch and have no limit. The
 * array holds 16 frames x 24 KiB of
 * transition operands plus 160 bytes of flags per head: 12 MiB + 5 KiB,
 * reserved on each device when the library's device code is loaded there,
 * whether or not this entry point is called. The first call on a device looks
 * the array's address up (cudaGetSymbolAddress, with that device current) and
 * keeps it for later calls; every call then clears the array's flags with
 * cudaMemsetAsync on `stream` before its kernel.
 *
 * Concurrency: every call on a device uses the same array. Two calls whose
 * work overlaps on the GPU (different streams with no ordering between them,
 * or calls from several host threads) race on it: their results are wrong or
 * a bounded device wait runs out (gdn_device_status then reports
 * GDN_ERR_TIMEOUT). Order such calls, on one stream or with events.
 * gdn_frame_scan and the other entry points do not touch the array.
 *
 * Arguments, layouts, results and errors are those of gdn_frame_scan; for
 * the same inputs and kernel choice (gdn_plan) the results are identical. */
#define GDN_NOALLOC_MAX_HEADS 32
GDN_API int gdn_frame_scan_noalloc(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int T, int S, int D, void* stream);

/* float32 variants: q, k, v, out are float; every operation runs in fp32 on
 * CUDA cores (FFMA), in the definition's order (W, then R, then K^T R). */
GDN_API int gdn_frame_scan_f32(const float* q, const float* k, const float* v,
                       const float* gamma, const float* beta,
                       const float* state_in, float* state_out, float* out,
                       int B, int H, int T, int S, int D, void* stream);

GDN_API int gdn_frame_step_f32(const float* q, const float* k, const float* v,
                       const float* gamma, const float* beta,
                       const float* state_in, float* state_out, float* out,
                       int B, int H, int S, int D, void* stream);

/* Variants with a `flags` word (0 gives exactly the calls above).
 *
 * GDN_FLAG_NO_DELTA: the update without the delta-rule correction, R = V_t:
 *     M_t = gamma_t M_{t-1} + beta_t (s K_t)^T V_t,   O_t = Q_t M_t.
 * This is the decayed cumulative state of block-causal linear attention, the
 * block KV cache of SANA-Video ("SANA-Video" ICLR 2026 oral transcript,
 * shadowingenglish.com, the part on block causal linear attention). With
 * gamma = beta = 1 it is plain cumulative linear attention over the frames
 * so far. Same kernels, layouts and precision as the delta-rule calls.
 * Any other bit returns GDN_ERR_FLAGS. */
#define GDN_FLAG_NO_DELTA 1u
GDN_API int gdn_frame_scan_ex(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int T, int S, int D, unsigned int flags, void* stream);
GDN_API int gdn_frame_step_ex(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int S, int D, unsigned int flags, void* stream);
GDN_API int gdn_frame_scan_f32_ex(const float* q, const float* k, const float* v,
                       const float* gamma, const float* beta,
                       const float* state_in, float* state_out, float* out,
                       int B, int H, int T, int S, int D, unsigned int flags, void* stream);
GDN_API int gdn_frame_step_f32_ex(const float* q, const float* k, const float* v,
                       const float* gamma, const float* beta,
                       const float* state_in, float* state_out, float* out,
                       int B, int H, int S, int D, unsigned int flags, void* stream);

/* Causal temporal convolution with a carried last-frame cache, the companion
 * of the GDN state in chunk-causal rollout ("SANA-Video" ICLR 2026 oral
 * transcript, shadowingenglish.com, the part on the causal FFN with temporal
 * convolution: a zero token is padded between two blocks so that a block
 * cannot see the next one, and the last token of a block is cached as the
 * first token the next block sees). Three depthwise taps along the frame
 * axis, centred on the current frame. Per channel c, token s, frame t, with
 * blocks of frames_per_block frames counted from the call's first frame:
 *
 *     y[t] = w[c][0] x_prev + w[c][1] x[t] + w[c][2] x_next + bias[c]
 *
 *   x_prev = x[t-1]; for t = 0, cache_in (the previous call's last frame;
 *            NULL means zero, the start of a video)
 *   x_next = x[t+1] inside a block; 0 for the last frame of a block (and of
 *            the call)
 *
 * cache_out receives x[T-1] (NULL: not written), so consecutive calls over
 * whole blocks equal one call. Layouts: x, y [B][T][S][C] bf16; w [C][3] and
 * bias [C] (or NULL) fp32; cache_in, cache_out [B][S][C] bf16. Arithmetic in
 * fp32, y rounded to bf16 (nearest even). C must be a multiple of 8
 * (GDN_ERR_SHAPE); x, y and the caches 16-byte aligned, w and bias 4-byte
 * aligned (GDN_ERR_ALIGN); y must not overlap x or the caches, cache_out must
 * not overlap x, and cache_in may equal cache_out (GDN_ERR_ALIAS). Device
 * pointers, stream-ordered like the other calls; allocates nothing. */
GDN_API int gdn_temporal_conv(const void* x, const float* w, const float* bias,
                              const void* cache_in, void* cache_out, void* y,
                              int B, int T, int S, int C, int frames_per_block, void* stream);

/* 3D rotary position embedding of queries or keys, applied before the scan
 * ("SANA-Video" ICLR 2026 oral transcript, shadowingenglish.com: 3D RoPE for
 * the linear attention). The talk gives no layout; this library's reading:
 * the head dimension D is cut into contiguous sections for the frame axis t,
 * the grid-row axis h and the grid-column axis w, of 2*floor(D/6) dims for h
 * and for w and the rest for t (D = 64: 24 + 20 + 20; D = 128: 44 + 42 + 42).
 * Inside a section of D_a dims, dims (2i, 2i+1) form pair i and turn
 * counter-clockwise by p * 10000^(-2i / D_a), p the token's position on that
 * axis: t0 + tau for the tau-th frame of the call, and for token r of a frame
 * on a grid grid_w tokens wide, h = r / grid_w and w = r % grid_w.
 *
 * x, y: [B][H][T][S][D] bf16, 16-byte aligned; y may equal x (in place), else
 * they must not overlap. The angle is p * freq in fp32 (freq from double),
 * cos and sin by sincosf, the rotation in fp32, y rounded to bf16 (nearest
 * even). D in {32, 64, 128}; grid_w >= 1; t0 >= 0. Allocates nothing. */
GDN_API int gdn_rope3d(const void* x, void* y, int B, int H, int T, int S, int D, int grid_w,
                       int t0, void* stream);

/* gdn_frame_step with 3D RoPE fused into its frame load: the row-split kernel
 * turns the frame's Q and K rows in shared memory as they arrive (the layout
 * of gdn_rope3d, frame position frame_index, grid grid_w tokens wide), before
 * any contraction reads them, so the rotated q and k never travel to HBM.
 * The result equals gdn_rope3d on q and on k followed by gdn_frame_step_ex,
 * bit for bit. Takes the sizes the row-split kernel takes (gdn_plan reports
 * GDN_KERNEL_STEP: D = 64, S <= 1408), else GDN_ERR_UNSUPPORTED; flags as in
 * gdn_frame_step_ex. grid_w >= 1 and frame_index >= 0 (else GDN_ERR_SHAPE). */
GDN_API int gdn_frame_step_rope(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int S, int D, int grid_w, int frame_index,
                   unsigned int flags, void* stream);

/* Chunk-causal streaming without a launch per frame: one persistent launch of
 * the row-split single-frame kernel (gdn_frame_step) serves frames from a
 * device-side frame queue as they are posted, keeping every head's D x D
 * state on chip between frames ("NVIDIA Apresenta SANA-WM ...",
 * acheiumaia.com.br: the chunk-causal autoregressive generator for
 * sequential rollout; one latent frame per recurrent step, constant state).
 *
 * The queue: rings of `ring` frame slots in device memory,
 *   q, k, v, out   [ring][B][H][S][D] bf16      gamma, beta  [ring][B][H] fp32,
 * and two counters in host memory mapped into the device (pinned host memory;
 * pass the device view, which under unified addressing is the host address):
 *   posted  written by the caller: frames 0 .. posted-1 are in their slots
 *           (frame n in slot n % ring). Setting bit 63 asks the kernel to stop
 *           once the posted frames are done.
 *   done    written by the kernel: frames 0 .. done-1 are complete for every
 *           head (their out slots are written).
 * queue_words: device memory, ring + 2 unsigned ints, 8-byte aligned, zero at
 * the call: the kernel's relay of `posted` (one CTA reads the host counter
 * and copies it there for the others to poll in device memory), then a count
 * per slot of the CTAs done with its frame (put back to zero after each frame).
 * Keep `posted` and `done` in different 128-byte lines: the host polls one
 * while the device reads the other.
 * The caller must fill slot n % ring before posting frame n, and must not
 * refill a slot before `done` has passed the frame it held. Frames are
 * processed in order; the state is read from state_in (NULL: zero) at the
 * start and written to state_out (NULL: not written) when the kernel stops.
 *
 * The call enqueues the launch on `stream` and returns; the kernel runs until
 * stopped. Its wait for the next frame is bounded by idle_timeout_ns: if
 * neither a frame nor the stop arrives in time it stops early and
 * gdn_device_status() reports GDN_ERR_TIMEOUT. Only host writes to `posted`
 * (and copies by the copy engines) may feed it: work on the same GPU that the
 * caller waits for before posting could find no free SM while the kernel
 * holds them. Launch it on a non-blocking stream, and while it runs issue no
 * work that CUDA's implicit synchronisation could order after it (work on the
 * legacy default stream, device or pinned allocations): the caller would
 * wait for a launch that waits for the caller, until the idle bound. Sizes: those of the row-split kernel (D = 64, S <= 1408) with
 * every head's cluster resident at once (B * H up to about 33 on a B200), else
 * GDN_ERR_UNSUPPORTED. Update and precision as gdn_frame_step; flags as in
 * gdn_frame_step_ex. Allocates nothing. */
GDN_API int gdn_frame_stream(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int S, int D, int ring,
                   const unsigned long long* posted, unsigned long long* done,
                   unsigned int* queue_words, unsigned long long idle_timeout_ns,
                   unsigned int flags, void* stream);

/* gdn_frame_stream with 3D RoPE (as gdn_frame_step_rope; "SANA-Video" ICLR
 * 2026 oral transcript, shadowingenglish.com: 3D RoPE for the linear
 * attention): every CTA turns its rows of q and k in shared memory as a
 * frame's tiles land, frame n of the queue (slot n % ring) as frame index
 * t0 + n on a grid grid_w tokens wide. The result equals a chain of
 * gdn_frame_step_rope calls with frame_index t0, t0 + 1, ... bit for bit.
 * D = 64; grid_w >= 1 and t0 >= 0 (else GDN_ERR_SHAPE); otherwise as
 * gdn_frame_stream. Allocates nothing. */
GDN_API int gdn_frame_stream_rope(const void* q, const void* k, const void* v,
                   const float* gamma, const float* beta,
                   const float* state_in, float* state_out, void* out,
                   int B, int H, int S, int D, int ring,
                   const unsigned long long* posted, unsigned long long* done,
                   unsigned int* queue_words, unsigned long long idle_timeout_ns,
                   int grid_w, int t0, unsigned int flags, void* stream);

/* Which kernel a bf16 call with these sizes runs, without running it.
 * Writes the kernel id (GDN_KERNEL_*) and the number of CTAs per head
 * (the thread-block cluster size, 1 for the CUDA-core kernel).
 * Returns GDN_OK or the error the call itself would return for the sizes. */
#define GDN_KERNEL_SIMT 1   /* CUDA-core kernel, one CTA per 16 state columns */
#define GDN_KERNEL_TC 2     /* tcgen05 kernel, a cluster of CTAs per head */
#define GDN_KERNEL_STEP 3   /* single-frame tcgen05 kernel (T = 1, D = 64): a cluster of
                               CTAs per head splits the frame's rows */
GDN_API int gdn_plan(int B, int H, int T, int S, int D, int* kernel, int* ctas_per_head);

/* Synchronizes the current device, then returns GDN_ERR_TIMEOUT if any kernel
 * since the last call recorded a wait that ran out (and clears the record),
 * GDN_ERR_CUDA if the synchronize failed, else GDN_OK. */
GDN_API int gdn_device_status(void);

/* Static text for a gdn_status value. Never NULL. */
GDN_API const char* gdn_status_string(int status);

/* GDN_VERSION_MAJOR * 10000 + GDN_VERSION_MINOR * 100 + GDN_VERSION_PATCH */
GDN_API int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBGDN_GDN_H_ */
