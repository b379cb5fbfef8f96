/*
 * fr.h -- C ABI of the B200 flow-matching action-expert denoising loop.
 *
 * The library runs the K-step Euler loop x <- x + dt * v(x, t) of a
 * π0.5-style action expert on one GPU.  v comes from an L-layer gated
 * transformer whose action tokens attend to a per-layer prefix KV cache that
 * is written once and reused by every step.
 *
 * Shape of the boundary (sources):
 *   - FlashRT walkthrough (m.lqnn.cn), component 7 "CUDA Graph capture": the
 *     hot forward takes device pointers only and allocates nothing.
 *   - same page, "exec/: C ABI execution contract": named device buffers are
 *     the only state (KV cache, scales, noise); cold start (load, calibrate)
 *     is separate from the hot call.
 *   - same page, section comparing with TensorRT/vLLM/SGLang: the KV cache is a
 *     static per-layer device buffer.
 *   - APXInf page ("Thor 芯片上，Pi0.5推理被干到了26ms"), section "一次跑得快，
 *     还要持续跑得稳": a fixed execution path with all memory allocated up front.
 *
 * Conventions
 *   - Every call returns FR_OK (0) or a negative FR_ERR_* code and never throws.
 *     The text of the last error of the calling thread is in fr_last_error().
 *   - A handle is not thread-safe.  It owns every device buffer it allocates;
 *     all device memory is allocated in fr_create and freed in fr_destroy.
 *   - Pointers passed in are borrowed: host pointers for the duration of the
 *     call, device pointers until the work queued on `stream` has finished.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     that take a stream are asynchronous unless stated otherwise.
 *   - A call on a handle that does device work first makes the handle's device
 *     (fr_create's `device`) the calling thread's current device, and leaves it
 *     current; `stream` must belong to that device, and device pointers passed
 *     in must point to its memory (the library does not enable peer access).
 *   - Device-side failures (a bounded wait that gave up, a device bounds check)
 *     are latched in a device status word; fr_sync_status() reads and clears it.
 */
#ifndef FR_H_
#define FR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fr_stream_t;   /* same type as cudaStream_t */
typedef struct fr_handle fr_handle;

enum {
  FR_OK = 0,
  FR_ERR_ARG = -1,          /* NULL pointer, negative size, bad enum */
  FR_ERR_SHAPE = -2,        /* B > B_max, P > P_max, sizes that do not fit the config */
  FR_ERR_STATE = -3,        /* e.g. denoise before weights / prefix, fp8 without scales */
  FR_ERR_CUDA = -4,         /* a CUDA runtime call failed (message has the CUDA error) */
  FR_ERR_TIMEOUT = -5,      /* a bounded device wait gave up */
  FR_ERR_DEVICE = -6,       /* a device-side bounds check failed */
  FR_ERR_UNSUPPORTED = -7   /* configuration outside what the kernels implement */
};

enum { FR_DTYPE_F32 = 0, FR_DTYPE_BF16 = 1, FR_DTYPE_FP8 = 2, FR_DTYPE_W4A16 = 3 };

/* Input features per scale group of the 4-bit weights of FR_DTYPE_W4A16. */
#define FR_W4_GROUP 128

/* Kernel set used by fr_denoise.  FR_PATH_AUTO picks the tensor-core path for
 * bf16/fp8/w4a16 and the CUDA-core path for f32.  FR_PATH_STEPWISE forces the simple
 * one-kernel-per-operation CUDA-core path (used by fp8 calibration as well). */
enum { FR_PATH_AUTO = 0, FR_PATH_STEPWISE = 1, FR_PATH_TENSOR = 2 };

/* What a handle runs (fr_config.role).  FR_ROLE_EXPERT: the denoising loop (fr_denoise).
 * FR_ROLE_PREFIX: the prefix pass (fr_prefill), the backbone whose per-layer keys and values
 * are the expert's prefix KV cache; there H is the largest number of prefix tokens per sample,
 * A, K and the time fields are unused (any valid value), dtype is bf16 or w4a16. */
enum { FR_ROLE_EXPERT = 0, FR_ROLE_PREFIX = 1 };

/* Flags of fr_set_prefix_kv. */
#define FR_PREFIX_K_ROTATED 1u   /* prefix K already carries RoPE at positions 0..P-1 */

/*
 * Sizes of one action expert.  Architecture per the workload descriptions:
 * pre-norm RMSNorm (eps), fused QKV projection, grouped-query attention with
 * rotate-half RoPE (rope_theta), merged gate|up projection with GeLU(tanh) on
 * the gate, sinusoidal time embedding (time_dim, time_base) fed through
 * Linear-SiLU-Linear and added to the in-projected action tokens.
 */
typedef struct fr_config {
  int L;          /* layers */
  int D;          /* width */
  int Hq, Hkv;    /* query heads, key/value heads (Hq % Hkv == 0) */
  int dh;         /* head dim (even) */
  int F;          /* MLP width of gate and of up */
  int H;          /* action tokens per chunk */
  int A;          /* action dim */
  int B_max;      /* largest batch fr_denoise will see */
  int P_max;      /* largest prefix length */
  int K;          /* Euler steps from t=1 to t=0, dt = -1/K */
  int dtype;      /* FR_DTYPE_* of the layer projections */
  int path;       /* FR_PATH_* */
  float rope_theta;
  float eps;
  int time_dim;
  float time_base;
  int adarms;     /* 0: the time embedding is added to the action tokens; 1: it conditions every
                     RMSNorm (adaptive RMSNorm, see fr_layer_weights.w_mod1) */
  int role;       /* FR_ROLE_* (0: the denoising loop) */
} fr_config;

/* Host float32 weights of one layer, row-major [out][in] (the nn.Linear convention). */
typedef struct fr_layer_weights {
  const float* wq;   /* [Hq*dh][D]  */
  const float* wk;   /* [Hkv*dh][D] */
  const float* wv;   /* [Hkv*dh][D] */
  const float* wo;   /* [D][Hq*dh]  */
  const float* wg;   /* [F][D] gate */
  const float* wu;   /* [F][D] up   */
  const float* wd;   /* [D][F] down */
  const float* g1;   /* [D] pre-attention RMSNorm gain (ignored and may be NULL when adarms) */
  const float* g2;   /* [D] pre-MLP RMSNorm gain (ignored and may be NULL when adarms) */
  /* adarms handles only (NULL otherwise).  The time embedding c of the step (the time MLP's
   * output) gives each norm (scale s, shift b, gate g) = w_mod c + b_mod, rows [s | b | g];
   * the norm's output is RMS(h) * (1 + s) + b and the residual update it feeds is scaled by g
   * (pi0.5-style adaptive RMSNorm; the pages do not describe the conditioning). */
  const float* w_mod1;   /* [3D][D] pre-attention norm */
  const float* b_mod1;   /* [3D] */
  const float* w_mod2;   /* [3D][D] pre-MLP norm */
  const float* b_mod2;   /* [3D] */
} fr_layer_weights;

/* Host float32 weights of the action expert, by name. */
typedef struct fr_weights {
  const fr_layer_weights* layers;   /* L entries */
  const float* w_in;   /* [D][A] */
  const float* b_in;   /* [D] */
  const float* w_out;  /* [A][D] */
  const float* b_out;  /* [A] */
  const float* w_t1;   /* [D][time_dim] */
  const float* b_t1;   /* [D] */
  const float* w_t2;   /* [D][D] */
  const float* b_t2;   /* [D] */
  const float* g_f;    /* [D] final RMSNorm gain (ignored and may be NULL when adarms) */
  const float* w_modf; /* adarms only: [2D][D] final norm modulation, rows [scale | shift] */
  const float* b_modf; /* adarms only: [2D] */
} fr_weights;

/*
 * fr_create -- validate the config, make `device` current and allocate ALL
 * device memory of the handle: packed weights, the KV cache
 * [L][B_max][Hkv][P_max+H][dh], activations, workspaces and status words.
 * Errors: FR_ERR_ARG (NULL, a size below 1, an unknown dtype, path or role),
 * FR_ERR_UNSUPPORTED (sizes the kernels do not implement), FR_ERR_CUDA
 * (allocation).  *out is NULL on error.
 */
int fr_create(const fr_config* cfg, int device, fr_handle** out);

/*
 * fr_load_weights -- pack host float32 weights into the handle
 * (PhyAI page, optimisation paragraph: Q/K/V fused into one GEMM, gate and up
 * merged; FlashRT walkthrough, component 4: declarative weight loading with
 * transpose/fuse/FP8-quantise transforms).  The packer concatenates
 * W_qkv = [W_q; W_k; W_v] and W_gu = [W_gate; W_up], rounds to bf16 (RNE) or,
 * for FR_DTYPE_FP8, quantises each fused projection to e4m3 with
 * s_w = max|w| / 448, or, for FR_DTYPE_W4A16, quantises every layer projection
 * to 4-bit codes with a bf16 scale per FR_W4_GROUP inputs (fr_quantize_w4), and
 * precomputes the K time embeddings and the RoPE tables.  For adarms handles it also
 * precomputes every step's norm modulation and folds each shift b into the projection it
 * feeds (W b added to that projection's output; the projection input is RMS(h) * (1 + s)).
 * Synchronous with respect to the host pointers; the caller keeps
 * ownership of `w`.  Errors: FR_ERR_ARG, FR_ERR_CUDA.
 */
int fr_load_weights(fr_handle* h, const fr_weights* w, fr_stream_t stream);

/*
 * fr_set_prefix_kv -- copy the per-layer prefix keys/values into the static KV
 * cache (FlashRT walkthrough: static per-layer KV buffers, computed once and
 * reused).  k_dev, v_dev: device [L][B][P][Hkv][dh], float32 for FR_DTYPE_F32
 * handles and bf16 otherwise.  Unless FR_PREFIX_K_ROTATED is set, K is rotated
 * at positions 0..P-1 on the way in.  The prefix stays until replaced.
 * Errors: FR_ERR_ARG, FR_ERR_SHAPE (B > B_max, P > P_max, P < 1), FR_ERR_CUDA.
 */
int fr_set_prefix_kv(fr_handle* h, const void* k_dev, const void* v_dev, int B, int P,
                     unsigned flags, fr_stream_t stream);

/*
 * fr_calibrate -- FP8 measure pass (FlashRT walkthrough, component 6, stage
 * (a)): run the whole K-step loop once on (x0_dev, prefix) with e4m3 weights
 * dequantised and projection inputs unquantised, record max|a| of each of the
 * 4 projection inputs of every layer over all steps, tokens and samples, then
 * set s_a = amax / 448 and alpha = s_a * s_w (stage (b)).  The calibration
 * prefix replaces the handle's prefix KV: call fr_set_prefix_kv afterwards.
 * Synchronises `stream`.  Errors: FR_ERR_STATE (not an fp8 handle, no
 * weights), FR_ERR_SHAPE, FR_ERR_CUDA.
 */
int fr_calibrate(fr_handle* h, const float* x0_dev, const void* pk_dev, const void* pv_dev,
                 int B, int P, fr_stream_t stream);

/*
 * fr_denoise -- the hot call: run K Euler steps on B chunks.
 * x0_dev: device float32 [B][H][A] noise at t=1; x_out_dev: device float32
 * [B][H][A] actions at t=0 (may alias x0_dev).  Asynchronous on `stream`,
 * allocates nothing.  Errors: FR_ERR_ARG, FR_ERR_SHAPE (B > B_max or B < 1),
 * FR_ERR_STATE (no weights, no prefix for these B samples, fp8 without
 * scales), FR_ERR_CUDA.  Device-side failures surface in fr_sync_status.
 */
int fr_denoise(fr_handle* h, const float* x0_dev, float* x_out_dev, int B, fr_stream_t stream);

/*
 * fr_get_scales / fr_set_scales -- export/import FP8 calibration.
 * s_act: host [L][4] activation scales in the order (qkv input, o input,
 * gate|up input, down input); s_w: host [L][4] weight scales, same order
 * (may be NULL).  n must be L*4.  fr_set_scales also recomputes alpha.
 * Errors: FR_ERR_ARG (NULL, a scale that is not positive and finite),
 * FR_ERR_SHAPE (n != L*4), FR_ERR_STATE (not fp8, no weights for set, scales
 * not set for get), FR_ERR_CUDA.
 */
int fr_get_scales(const fr_handle* h, float* s_act, float* s_w, int n);
int fr_set_scales(fr_handle* h, const float* s_act, int n);

/*
 * fr_sync_status -- synchronise `stream`, read and clear the device status
 * word.  Returns FR_OK, FR_ERR_TIMEOUT or FR_ERR_DEVICE (message says where).
 */
int fr_sync_status(fr_handle* h, fr_stream_t stream);

/*
 * fr_selftest_wait -- failure-detection self-test: launches one kernel whose single device wait
 * (an mbarrier that nothing completes) gives up after limit_ns, exactly as a wait of the loop's
 * kernels does: it latches the timeout bit and the where-code 0x7F0 in the status word and the
 * kernel returns, leaving the context usable.  The next fr_sync_status returns FR_ERR_TIMEOUT
 * and clears the word.  No counterpart in the pages: it exists to test that path without
 * faulting or hanging the GPU.  limit_ns in [1 us, 100 ms].  Asynchronous.
 * Errors: FR_ERR_ARG (NULL, limit out of range), FR_ERR_CUDA.
 */
int fr_selftest_wait(fr_handle* h, uint64_t limit_ns, fr_stream_t stream);

/* Text of the last error on the calling thread ("" if none).  Never NULL. */
const char* fr_last_error(void);

/* Free every device buffer of the handle.  NULL is a no-op. */
void fr_destroy(fr_handle* h);

/* ---- introspection (verification and tooling; not on the hot path) ---- */

/*
 * fr_read_kv -- copy layer `layer`, sample `b` of the KV cache to host:
 * k_host, v_host receive [Hkv][n_slots][dh] in the cache's storage type
 * (float32 for f32 handles, bf16 bits otherwise), n_slots = P + H (prefix
 * slots first, then the action slots of the last step).  Synchronous.
 */
int fr_read_kv(const fr_handle* h, int layer, int b, void* k_host, void* v_host, int n_slots);

/* Copy the handle's RoPE tables [n_pos][dh/2] to host (n_pos <= P_max + H). */
int fr_get_rope_tables(const fr_handle* h, float* cos_host, float* sin_host, int n_pos);

/* Name of the kernel set fr_denoise runs ("stepwise" or "tensor"). */
const char* fr_path_name(const fr_handle* h);

/* Number of kernel launches one fr_denoise call (fr_prefill for a prefix handle) issues for batch B
 * at the current prefix length. */
int fr_launches_per_call(const fr_handle* h, int B);

/*
 * Execution of the tensor-core path (PhyAI page, profiling paragraph: at batch 1 the loop's time
 * goes to many small launches; optimisation paragraph: the ten-step Euler iteration replayed as
 * one unit).  FR_EXEC_PERSISTENT: one cooperative launch of a persistent kernel runs the whole
 * call, one CTA per SM, its phases handed over through bounded device-side waits; it serves bf16
 * handles without adaRMS whose calls have B*H <= 64 tokens.  FR_EXEC_GRAPH: one CUDA graph of
 * K*(2 + 5L) kernels chained by programmatic dependent launch, for every shape.  FR_EXEC_AUTO
 * (the default) replays the graph, which is the faster of the two as measured at pi0.5 batch 1.
 */
enum { FR_EXEC_AUTO = 0, FR_EXEC_GRAPH = 1, FR_EXEC_PERSISTENT = 2 };

/* fr_set_exec_mode -- choose FR_EXEC_*.  With FR_EXEC_PERSISTENT, fr_denoise returns
 * FR_ERR_UNSUPPORTED for calls the persistent kernel does not serve.  Errors: FR_ERR_ARG (NULL,
 * unknown mode), FR_ERR_STATE (not a tensor-path expert handle). */
int fr_set_exec_mode(fr_handle* h, int mode);

/* fr_exec_mode -- FR_EXEC_PERSISTENT or FR_EXEC_GRAPH: what a call of batch B at the current prefix
 * length runs; negative error code on a NULL handle or a handle off the tensor path. */
int fr_exec_mode(const fr_handle* h, int B);

/* fr_set_wait_limit -- bound, in ns, of every wait of the persistent kernel on work of another CTA
 * (0 restores the default, 2 s).  A wait that gives up latches FR_ERR_TIMEOUT in the status word
 * (fr_sync_status) and every CTA of the call leaves its loops and returns; the call's outputs are
 * then undefined and the next call starts afresh.  Errors: FR_ERR_ARG (NULL, limit above 10 s). */
int fr_set_wait_limit(fr_handle* h, uint64_t limit_ns);

/* ---- device bounds checks (checked builds) ---- */

/* 1 if this library was built with device bounds checks (-DFR_DEVICE_CHECKS), else 0.  In a checked
 * build every store of the GEMM epilogues, of the attention kernels and of the persistent kernel
 * verifies its index against its buffer's extent; an index at or past it latches FR_ERR_DEVICE in the
 * status word (fr_sync_status / fr_ops_sync_status: where-code and index) and the store is skipped.
 * No counterpart in the pages: it stands in for a memory checker in debugging. */
int fr_device_checks(void);

/* fr_debug_plan -- host only, no device: the tensor-core path's launch plan of one fr_denoise call of
 * batch B and prefix length P (for an FR_ROLE_PREFIX config: the pass over P tokens) on a device with
 * nsm SMs, max_dyn bytes of dynamic shared memory per CTA and max_dyn2 bytes per CTA when two share an
 * SM.  No counterpart in the pages: it lets the host logic that sizes every launch be tested without a
 * GPU.  out[0..n_out) receives: NT, Nt (token tiles, tokens per tile); then for the QKV, O, gate|up and
 * down projections in turn eight ints each: split-K S, ring slots, tokens per epilogue staging pass,
 * persistent kernel (0/1), k-chunks per ring slot, dynamic shared memory (bytes), tiles (m-blocks x NT),
 * k-chunks of 64 bf16 / 128 e4m3 inputs; then the attention kernel (1: tcgen05), its key chunks and keys
 * per chunk.  Returns the number of entries of the plan (37; fewer are written if n_out is smaller) or
 * FR_ERR_ARG, the configuration errors of fr_create, FR_ERR_UNSUPPORTED (outside the tensor-core
 * path), FR_ERR_SHAPE (B or P out of range). */
int fr_debug_plan(const fr_config* cfg, int B, int P, int nsm, int max_dyn, int max_dyn2, int* out, int n_out);

/* fr_debug_limit_extent -- checked builds: declare a smaller extent (elements of the buffer's type;
 * bytes for the tiled operands) for one of the handle's buffers "h", "q", "kv", "xbuf", "obuf",
 * "ubuf", "ssq" or "x" (0 restores the real one), so that the bounds checks can be exercised without
 * any access leaving the real allocation.  Cached graphs are dropped.  Errors: FR_ERR_ARG (NULL,
 * unknown name), FR_ERR_STATE (not a tensor-path handle), FR_ERR_UNSUPPORTED (not a checked build). */
int fr_debug_limit_extent(fr_handle* h, const char* buffer, uint64_t elems);

/*
 * fr_prefill -- the prefix pass, the step before the loop (FlashRT walkthrough, component 5:
 * the attention sites of the Pi0.5 model; the loop's per-layer KV cache is the backbone's keys and
 * values of the observation's tokens).  `backbone` is an FR_ROLE_PREFIX handle with weights (only
 * the layer tensors of fr_weights are read; the others may be NULL).  emb_dev: device bf16
 * [B][P][D] embedded prefix tokens (vision encoder and text embedding outputs).  Runs the
 * backbone's layers over the P tokens of each sample with full attention among them and RoPE
 * at positions 0..P-1 (one CUDA graph per (B, P); the last layer stops after its QKV
 * projection); every layer's rotated K and its V land in the backbone's KV cache (named buffers
 * "kv_k"/"kv_v", slots 0..P-1).  When `expert` is not NULL they are also copied into its prefix
 * KV for slots 0..B-1, which then holds (B, P) as after fr_set_prefix_kv with
 * FR_PREFIX_K_ROTATED; the expert needs the backbone's L, Hkv and dh and a bf16 KV cache.
 * Asynchronous on `stream`; allocates nothing.
 * Errors: FR_ERR_ARG (NULL, expert handle on another device), FR_ERR_STATE (not a prefix
 * handle, no weights, expert not an expert handle), FR_ERR_SHAPE (B > B_max, P > H of the
 * backbone or P_max of the expert, KV shapes differ), FR_ERR_CUDA.
 */
int fr_prefill(fr_handle* backbone, const void* emb_dev, int B, int P, fr_handle* expert, fr_stream_t stream);

/* ---- execution contract across chunks: selective refresh, named buffers, capsules ---- */

/*
 * fr_refresh_prefix_kv -- selective refresh of the prefix state (FlashRT-PAI overview,
 * mechanism 2 "execution contract": state reused across decision cycles and refreshed
 * only where it changed): replace the prefix KV of n batch slots and leave every other
 * slot as it is, e.g. when one camera's observation of a batch of robots changed.
 * k_dev, v_dev: device [L][n][P][Hkv][dh] in the type of fr_set_prefix_kv; source sample
 * i goes to slot slots[i] (host array of n distinct slots, each below the B of the last
 * fr_set_prefix_kv or fr_capsule_restore).  P must equal that call's P: the cache holds
 * one prefix length.  K is rotated at 0..P-1 unless FR_PREFIX_K_ROTATED.  Asynchronous.
 * Errors: FR_ERR_ARG (NULL, n < 1, a slot given twice, unknown flags), FR_ERR_STATE (no
 * prefix yet), FR_ERR_SHAPE (P differs, slot out of range), FR_ERR_CUDA.
 */
int fr_refresh_prefix_kv(fr_handle* h, const void* k_dev, const void* v_dev, const int* slots, int n, int P,
                         unsigned flags, fr_stream_t stream);

/*
 * fr_get_buffer -- a named device buffer of the handle (FlashRT walkthrough, "exec/: C
 * ABI execution contract": named device buffers are the only state and are shared by
 * pointer between graphs, without copies).  Names and contents:
 *   "kv_k", "kv_v"          KV cache [L][B_max][Hkv][P_max+H][dh], each layer starting on
 *                           a 256-byte boundary; float32 for f32 handles, bf16 otherwise
 *   "rope_cos", "rope_sin"  RoPE tables [P_max+H][dh/2] float32
 *   "temb"                  time embeddings of the K steps [K][D] float32
 *   "s_act"                 fp8 activation scales [L][4] float32 (see fr_get_scales)
 *   "status"                the device status word (uint32)
 * *dev receives the device address and *bytes the size; the handle owns both until
 * fr_destroy.  Writing into them is the caller's responsibility.  No device work.
 * Errors: FR_ERR_ARG (NULL argument, unknown name).
 */
int fr_get_buffer(const fr_handle* h, const char* name, void** dev, size_t* bytes);

/*
 * Execution-state capsules (FlashRT-PAI overview, mechanism 3: snapshot, restore and
 * fork of the resident pipeline state; FlashRT walkthrough, "serving/": snapshot,
 * restore, fork and time travel).  Between chunks the state of a handle is the prefix
 * KV of its batch slots; a capsule holds it for B samples, plus the caller's action
 * chunk x [B][H][A] float32 when saved with one.  The capsule's bytes live in a device
 * buffer the caller owns; the fr_capsule description stays on the host.
 * Device layout: K [L][B][Hkv][P][dh], then V in the same layout, then x; each part
 * starts on a 256-byte boundary; K/V in the KV cache's type (K already rotated).
 */
#define FR_CAPSULE_MAGIC 0x46524350u
typedef struct fr_capsule {
  uint32_t magic;          /* FR_CAPSULE_MAGIC once written by fr_capsule_save */
  int L, Hkv, dh;          /* shape of the handle that wrote it */
  int kv_bytes_per_elem;   /* 2 (bf16) or 4 (float32) */
  int H, A;
  int B, P;                /* samples and prefix length held */
  int has_x;               /* 1: x [B][H][A] follows the KV */
  size_t bytes;            /* device bytes in use */
} fr_capsule;

/* Device bytes of a capsule of B samples and prefix length P (with x when with_x != 0)
 * for handles created from *cfg; 0 if cfg is invalid, B outside [1, B_max] or P outside
 * [1, P_max].  Host arithmetic only. */
size_t fr_capsule_bytes(const fr_config* cfg, int B, int P, int with_x);

/*
 * fr_capsule_save -- snapshot the prefix KV of slots 0..B-1 (B at most the cached batch)
 * and, when x_dev is not NULL, the chunk x_dev [B][H][A] into cap_dev, a device buffer of
 * cap_bytes >= fr_capsule_bytes(cfg, B, P, x_dev != NULL) bytes.  *desc receives the
 * description.  Asynchronous: the snapshot is the state at this point of `stream`.
 * Errors: FR_ERR_ARG (NULL), FR_ERR_STATE (no prefix yet), FR_ERR_SHAPE (B, cap_bytes),
 * FR_ERR_CUDA.
 */
int fr_capsule_save(const fr_handle* h, void* cap_dev, size_t cap_bytes, int B, const float* x_dev,
                    fr_capsule* desc, fr_stream_t stream);

/*
 * fr_capsule_restore -- make a capsule the handle's prefix state: slot b (b < B) receives
 * capsule sample map[b] (map NULL: sample b, then B <= desc->B).  A map that repeats a
 * sample forks it into several slots (several noise draws against one observation).  A
 * capsule saved earlier brings back an earlier state.  Afterwards the cached prefix covers
 * slots 0..B-1 with length desc->P, as after fr_set_prefix_kv.  When x_dev is not NULL,
 * x_dev [B][H][A] receives the capsule's x of the same samples.  Asynchronous.
 * Errors: FR_ERR_ARG (NULL, not a capsule description, map entry out of range),
 * FR_ERR_SHAPE (capsule of a handle of another shape, B outside [1, B_max], desc->P >
 * P_max, B > desc->B without a map), FR_ERR_STATE (not an expert handle; x_dev given,
 * capsule without x), FR_ERR_CUDA.
 */
int fr_capsule_restore(fr_handle* h, const void* cap_dev, const fr_capsule* desc, const int* map, int B,
                       float* x_dev, fr_stream_t stream);

/*
 * fr_set_graph_capacity / fr_graph_count -- the tensor path keeps one instantiated CUDA
 * graph per (B, P) it has run (FlashRT walkthrough, "exec/": shape key -> graph variant,
 * exact key, least recently used evicted).  At most `capacity` (>= 1; 8 at fr_create)
 * stay; the least recently used goes first, a graph still running being freed once it
 * completes.  fr_graph_count returns how many are cached (0 on the stepwise path).
 * Errors: FR_ERR_ARG (NULL, capacity < 1).
 */
int fr_set_graph_capacity(fr_handle* h, int capacity);
int fr_graph_count(const fr_handle* h);

/* ---- kernel library: one op on caller buffers (no handle) ---- */

/*
 * fr_attention -- the loop's split-KV grouped-query attention as a stand-alone op
 * (FlashRT walkthrough, component 5: the Pi0.5 decoder attention site; component 8:
 * a kernel library with a stable op ABI).  For every sample b, query head j and query
 * row i:  o = softmax(q k^T / sqrt(dh)) v  over all S_keys keys of KV head
 * floor(j * Hkv / Hq); no mask.
 * q: device bf16 [B][Hq][H][dh]; k, v: device bf16 [B][Hkv][S_keys][dh] (keys already
 * rotated); o: device bf16 [B][H][Hq*dh] (row-major, the O-projection input layout).
 * Keys are split into up to 16 chunks of a multiple of 64 keys; the chunks' partial rows
 * are merged through `scratch`, a device buffer of fr_attention_scratch_bytes() bytes
 * owned by the caller (NULL when that size is 0).  Asynchronous on `stream`.
 * Limits: dh in {64, 128, 256}, Hq % Hkv == 0, 1 <= H <= 128, H <= S_keys <= 32768.
 * Errors: FR_ERR_ARG (NULL pointer, bad size), FR_ERR_UNSUPPORTED (limits),
 * FR_ERR_SHAPE (scratch smaller than needed), FR_ERR_CUDA.  A device wait of the op that
 * gives up (see fr_sync_status) is latched in the ops' status word of the device: read it
 * with fr_ops_sync_status.
 */
int fr_attention(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int H, int S_keys,
                 int dh, void* scratch, size_t scratch_bytes, fr_stream_t stream);

/*
 * fr_ops_sync_status -- synchronise `stream`, then read and clear the status word that the
 * stand-alone ops (fr_attention, fr_attention_noalloc) of the current device latch their
 * device-side failures in.  Returns FR_OK, FR_ERR_TIMEOUT (the message gives the wait's
 * where-code and block) or, in a checked build, FR_ERR_DEVICE (a store's index failed its
 * bounds check: where-code and index).  The word is one per device, shared by every op call
 * on it.
 * Errors: FR_ERR_CUDA.
 */
int fr_ops_sync_status(fr_stream_t stream);

/* Bytes of scratch fr_attention needs for these sizes (0 if the keys fit one chunk). */
size_t fr_attention_scratch_bytes(int B, int Hq, int H, int S_keys, int dh);

/* Bytes of the scratch array built into the library for fr_attention_noalloc. */
#define FR_ATTENTION_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * fr_attention_noalloc -- fr_attention without a scratch argument.  The paper has no
 * counterpart: it is a convenience of this library.  It serves callers that cannot
 * allocate or own a device buffer: a control loop that must not enter an allocator once it
 * runs (cudaMalloc may synchronise the device and takes unbounded time), a plug-in handed
 * tensors but no workspace by its host framework, or code that must not change its device
 * memory footprint after start-up.  For them the chunk-merge scratch is one fixed device
 * array inside the library, FR_ATTENTION_NOALLOC_SCRATCH_BYTES (8 MiB) per device; this
 * function allocates nothing.
 * Arguments, layouts, limits and errors are those of fr_attention; in addition sizes whose
 * fr_attention_scratch_bytes() exceeds the array are rejected with FR_ERR_UNSUPPORTED
 * (the π0.5 layer shape, B=1 Hq=8 H=50 S_keys=866 dh=256, needs 5.8 MB).
 * The first call on a device looks up the array's address on that device (and sets the
 * kernel attributes); make that first call before any stream capture that should contain
 * later calls.  All calls on one device share the one array: two calls whose kernels can
 * overlap in time (different streams, or different host threads without ordering) race
 * on it and may return wrong results; calls ordered on one stream are safe.  The array
 * needs no clearing: each launch writes every word it reads before reading it.  Device-side
 * failures go to the ops' status word (fr_ops_sync_status).
 */
int fr_attention_noalloc(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int H,
                         int S_keys, int dh, fr_stream_t stream);

/* ---- host number-format utilities used by the packer (no GPU needed) ---- */

/* RoPE tables: cos/sin of pos * theta^(-2j/dh) for pos < n_pos, j < dh/2, float64
 * math rounded once to float32 (rotate-half pairing (j, j + dh/2)). */
int fr_rope_tables(int n_pos, int dh, double theta, float* cos_out, float* sin_out);

/* float32 -> bf16 bits, round to nearest even (NaN stays NaN). */
void fr_round_bf16(const float* in, uint16_t* out, size_t n);

/* 4-bit group quantisation of a row-major [rows][cols] float32 weight (FR_DTYPE_W4A16;
 * PhyAI page, optimisation paragraph: W4A16; the group size is this library's reading).
 * Per row and per group of FR_W4_GROUP consecutive columns: scale s = bf16(max|w| / 7),
 * one rounding from float64, returned as bf16 bits in scale_bits [rows][ceil(cols/128)];
 * codes q = round-half-even(w / s) clamped to [-7, 7] in q [rows][cols]; an all-zero group
 * has s = 0 and q = 0.  The projection uses bf16(q * s).  FR_ERR_ARG on NULL or negative sizes. */
int fr_quantize_w4(const float* w, int rows, int cols, int8_t* q, uint16_t* scale_bits);

/* float32 -> e4m3 bytes of in[i] / scale computed in float64: saturate to +-448,
 * round to nearest even (OCP E4M3, no infinities, NaN -> 0x7F). */
void fr_quantize_e4m3(const float* in, uint8_t* out, size_t n, double scale);

#ifdef __cplusplus
}
#endif

#endif /* FR_H_ */
