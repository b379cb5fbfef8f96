// Kernel-library entry points: one op of the loop on caller-owned device buffers.
//
// FlashRT walkthrough, component 8: the kernel library exposes its ops through a stable
// ABI, separate from the per-model pipeline.  Here that is the split-KV grouped-query
// attention of the action tokens over [prefix; actions] (component 5: the Pi0.5 decoder
// attention site), the same kernel fr_denoise runs for every layer.
#include <cmath>
#include <mutex>

#include "internal.h"
#include "tc_kernels.h"

namespace fr {
namespace {

constexpr int MAX_DEVICES = 64;
std::once_flag g_init_once[MAX_DEVICES];
cudaError_t g_init_err[MAX_DEVICES];

}  // namespace

// Kernel attributes are per device; set them once on each device the ops run on.
cudaError_t ensure_tc_kernels(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::call_once(g_init_once[dev], [dev] { g_init_err[dev] = tc::tc_kernels_init(); });
  if (dev_out) *dev_out = dev;
  return g_init_err[dev];
}

namespace {

// Status word of the stand-alone ops ([0] flags, [1] where, [2] block, as a handle's): one per
// device (module globals are per context), its address looked up once per device.
static __device__ __align__(16) unsigned g_ops_status[4];

std::once_flag g_status_once[MAX_DEVICES];
unsigned* g_status_ptr[MAX_DEVICES];
cudaError_t g_status_err[MAX_DEVICES];

}  // namespace

// Device address of the ops' status word on the current device (kernel attributes set too).
cudaError_t ops_status_word(unsigned** out, int* dev_out) {
  int dev = 0;
  cudaError_t e = ensure_tc_kernels(&dev);
  if (e != cudaSuccess) return e;
  std::call_once(g_status_once[dev], [dev] {
    void* p = nullptr;
    g_status_err[dev] = cudaGetSymbolAddress(&p, g_ops_status);
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  });
  *out = g_status_ptr[dev];
  if (dev_out) *dev_out = dev;
  return g_status_err[dev];
}

int check_attention(const void* q, const void* k, const void* v, const void* o, int B, int Hq, int Hkv, int H,
                    int S_keys, int dh) {
  if (!q || !k || !v || !o) {
    set_error("fr_attention: NULL tensor");
    return FR_ERR_ARG;
  }
  if (B < 1 || Hq < 1 || Hkv < 1 || H < 1 || S_keys < 1) {
    set_error("fr_attention: sizes must be positive");
    return FR_ERR_ARG;
  }
  if ((dh != 64 && dh != 128 && dh != 256) || Hq % Hkv != 0 || H > 128 || H > S_keys || S_keys > 32768) {
    set_error("fr_attention: needs dh in {64,128,256}, Hq %% Hkv == 0, H <= 128, H <= S_keys <= 32768");
    return FR_ERR_UNSUPPORTED;
  }
  int C = 1, KC = 64;
  tc::attn_chunks(S_keys, C, KC);
  if (tc::attn_smem_bytes(H, dh, KC, C, 0) > 200 * 1024) {
    set_error("fr_attention: a key chunk of %d keys does not fit shared memory", KC);
    return FR_ERR_UNSUPPORTED;
  }
  return FR_OK;
}

tc::AttnArgs attention_args(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int H,
                            int S_keys, int dh, float* scratch, unsigned* status) {
  tc::AttnArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv_k = static_cast<const __nv_bfloat16*>(k);
  a.kv_v = static_cast<const __nv_bfloat16*>(v);
  a.o = static_cast<uint8_t*>(o);
  a.o_rowmajor = 1;
  a.fp8 = 0;
  a.H = H;
  a.P = S_keys - H;
  a.S_max = S_keys;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.dh = dh;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  a.umma = tc::attn_plan(S_keys, tc::attn_tiles(B, Hq, Hkv, H), nsm, a.C, a.KC);
  a.scale = 1.0f / std::sqrt(static_cast<float>(dh));
  a.xscratch = scratch;
  a.status = status;
  a.o_extent = static_cast<uint64_t>(B) * H * Hq * dh * 2;
  return a;
}

}  // namespace fr

using namespace fr;

extern "C" {

size_t fr_attention_scratch_bytes(int B, int Hq, int H, int S_keys, int dh) {
  if (B < 1 || Hq < 1 || H < 1 || S_keys < 1 || dh < 1) return 0;
  int C = 1, KC = 64;
  tc::attn_chunks(S_keys, C, KC);
  return tc::attn_scratch_bytes(B, Hq, C, H, dh);
}

int fr_attention(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int H, int S_keys,
                 int dh, void* scratch, size_t scratch_bytes, fr_stream_t stream) {
  int rc = check_attention(q, k, v, o, B, Hq, Hkv, H, S_keys, dh);
  if (rc) return rc;
  const size_t need = fr_attention_scratch_bytes(B, Hq, H, S_keys, dh);
  if (need > 0 && (!scratch || scratch_bytes < need)) {
    set_error("fr_attention: scratch of %zu bytes needed, %zu given", need, scratch ? scratch_bytes : size_t(0));
    return FR_ERR_SHAPE;
  }
  unsigned* status = nullptr;
  FR_CUDA(ops_status_word(&status, nullptr));
  const tc::AttnArgs a = attention_args(q, k, v, o, B, Hq, Hkv, H, S_keys, dh, static_cast<float*>(scratch), status);
  FR_CUDA(tc::launch_attention_tc(a, B, reinterpret_cast<cudaStream_t>(stream), false));
  return FR_OK;
}

int fr_ops_sync_status(fr_stream_t stream) {
  unsigned* status = nullptr;
  FR_CUDA(ops_status_word(&status, nullptr));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned st[4] = {0, 0, 0, 0};
  FR_CUDA(cudaMemcpyAsync(st, status, sizeof(st), cudaMemcpyDeviceToHost, s));
  FR_CUDA(cudaStreamSynchronize(s));
  FR_CUDA(cudaMemsetAsync(status, 0, sizeof(st), s));
  FR_CUDA(cudaStreamSynchronize(s));
  if (st[0] & ST_TIMEOUT) {
    set_error("device wait gave up in an op (phase word 0x%08x, block %u)", st[1], st[2]);
    return FR_ERR_TIMEOUT;
  }
  if (st[0] & ST_BOUNDS) {   // checked builds
    set_error("device bounds check failed in an op (where 0x%08x, index %u)", st[1], st[2]);
    return FR_ERR_DEVICE;
  }
  return FR_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- fr_attention_noalloc
// The same kernel with its chunk-merge scratch in a fixed array of this library's device
// image instead of a caller buffer.  Every device the library runs on holds its own copy
// of the array (module globals are per context); its address is looked up once per device.
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = FR_ATTENTION_NOALLOC_SCRATCH_BYTES;
static_assert(NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch array size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

std::once_flag g_noalloc_once[MAX_DEVICES];
void* g_noalloc_ptr[MAX_DEVICES];
cudaError_t g_noalloc_err[MAX_DEVICES];

}  // namespace

extern "C" int fr_attention_noalloc(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv,
                                    int H, int S_keys, int dh, fr_stream_t stream) {
  int rc = check_attention(q, k, v, o, B, Hq, Hkv, H, S_keys, dh);
  if (rc) return rc;
  const size_t need = fr_attention_scratch_bytes(B, Hq, H, S_keys, dh);
  if (need > NOALLOC_SCRATCH_BYTES) {
    set_error("fr_attention_noalloc: these sizes need %zu bytes of scratch; the built-in array holds %zu "
              "(call fr_attention with a caller-owned buffer instead)", need, NOALLOC_SCRATCH_BYTES);
    return FR_ERR_UNSUPPORTED;
  }
  int dev = 0;
  unsigned* status = nullptr;
  FR_CUDA(ops_status_word(&status, &dev));
  // once per device, with that device current: the array's device address
  std::call_once(g_noalloc_once[dev], [dev] {
    g_noalloc_err[dev] = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
  });
  if (g_noalloc_err[dev] != cudaSuccess) return cuda_fail(g_noalloc_err[dev], "cudaGetSymbolAddress(scratch)");
  // every scratch word the kernel reads is written earlier in the same launch: nothing to clear
  const tc::AttnArgs a =
      attention_args(q, k, v, o, B, Hq, Hkv, H, S_keys, dh, static_cast<float*>(g_noalloc_ptr[dev]), status);
  FR_CUDA(tc::launch_attention_tc(a, B, reinterpret_cast<cudaStream_t>(stream), false));
  return FR_OK;
}
