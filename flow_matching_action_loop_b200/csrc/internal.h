// Internal declarations of the action-expert library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <string>

#include "fr.h"

namespace fr {

// Quantisation applied where an activation is written as a projection input.
enum QMode : int {
  Q_NONE = 0,      // keep float32 (f32 workloads)
  Q_BF16 = 1,      // round to bf16 (R10)
  Q_E4M3 = 2,      // e4m3 code value of a / s_a (R11)
  Q_MEASURE = 3,   // keep float32 and record max|a| (fp8 calibration measure pass)
};

// Index of a projection input in the per-layer scale arrays.
enum ProjInput : int { PI_QKV = 0, PI_O = 1, PI_GU = 2, PI_DOWN = 3, PI_COUNT = 4 };

// Device status word bits (latched by kernels, read by fr_sync_status).
enum StatusBits : uint32_t {
  ST_TIMEOUT = 1u,
  ST_BOUNDS = 2u,
};

void set_error(const char* fmt, ...);
int cuda_fail(cudaError_t e, const char* what);

#define FR_CUDA(call)                                         \
  do {                                                        \
    cudaError_t e_ = (call);                                  \
    if (e_ != cudaSuccess) return ::fr::cuda_fail(e_, #call); \
  } while (0)

// ------------------------------------------------------------------ stepwise kernels
// (one kernel per operation, CUDA cores, float32 activations holding values already
// rounded to the projection-input grid; see stepwise.cu)

struct StepwiseWeights {      // one layer, row-major [out][in], storage type by dtype
  const void* wqkv;           // [(Hq+2Hkv)dh][D]
  const void* wo;             // [D][Hq dh]
  const void* wgu;            // [2F][D]  (gate rows then up rows)
  const void* wd;             // [D][F]
  const float* g1;
  const float* g2;
};

void launch_temb(const float* w_t1, const float* b_t1, const float* w_t2, const float* b_t2,
                 float* temb, int D, int time_dim, int K, float time_base, int round_bf16,
                 cudaStream_t s);
void launch_inproj(const float* x, const float* w_in, const float* b_in, const float* temb_k,
                   float* h, int T, int D, int A, int round_bf16, cudaStream_t s);
void launch_rmsnorm_q(const float* h, const float* gamma, float* out, int T, int D, float eps,
                      int qmode, const float* s_a, unsigned* amax, cudaStream_t s);
// C[t][n] (+)= gate[n] * alpha * (A W^T)[t][n] + bias[n]  (gate, bias: NULL = 1, 0)
void launch_gemm(const float* A, int lda, const void* W, int wtype, const float* alpha,
                 float* C, int ldc, int T, int N, int Kd, int accumulate, cudaStream_t s,
                 const float* bias = nullptr, const float* gate = nullptr);
void launch_round_rows(const float* in, int in_ld, float* out, int rows, int n, int round_bf16, cudaStream_t s);
void launch_one_plus(const float* in, int in_ld, float* out, int rows, int n, cudaStream_t s);
void launch_rope_qkv(const float* qkv, float* q, void* kv_k, void* kv_v, int kv_bf16,
                     const float* cos_t, const float* sin_t, int B, int H, int P, int S_max,
                     int Hq, int Hkv, int dh, int round_bf16, cudaStream_t s);
// Batch slots written by one prefix-ingest launch: source sample b0 + i goes to slot slot[i]
// (n == 0: slot b0 + i).
constexpr int SLOT_MAP_MAX = 64;
struct SlotMap {
  int n;
  int slot[SLOT_MAP_MAX];
};
// in [L][B_src][P][Hkv][dh] samples b0 .. b0+nb-1 -> cache [L][B_max][Hkv][S_max][dh]
void launch_prefix_ingest(const void* k_in, const void* v_in, void* kv_k, void* kv_v, int kv_bf16,
                          const float* cos_t, const float* sin_t, int L, int B_src, int b0, int nb,
                          const SlotMap& map, int B_max, int P, int S_max, int Hkv, int dh, int rotate,
                          cudaStream_t s);
void launch_attention(const float* q, const void* kv_k, const void* kv_v, int kv_bf16, float* act,
                      int ld_act, int B, int H, int P, int S_max, int Hq, int Hkv, int dh,
                      int qmode, const float* s_a, unsigned* amax, cudaStream_t s);
void launch_gelu_mul(const float* gu, float* act, int T, int F, int qmode, const float* s_a,
                     unsigned* amax, cudaStream_t s);
void launch_final(const float* h, const float* g_f, const float* w_out, const float* b_out,
                  float* x, int T, int D, int A, float eps, float dt, int round_bf16, cudaStream_t s);

enum WType : int { W_F32 = 0, W_BF16 = 1, W_E4M3 = 2 };

// ------------------------------------------------------------------ state copies (state.cu)
// Rows (outer, sample, mid, row) of row_bytes (a multiple of 4) copied for each of `parts`
// (src, dst) pairs; destination sample b (b < n_sample <= SLOT_MAP_MAX) reads source sample
// map[b].  Strides are in bytes.
struct RowCopy {
  const char* src[2];
  char* dst[2];
  int parts;
  long long n_outer, n_sample, n_mid, n_row;
  long long s_outer, s_sample, s_mid, s_row;
  long long d_outer, d_sample, d_mid, d_row;
  long long row_bytes;
  int row_words;   // set by the launcher
  int map[SLOT_MAP_MAX];
};
void launch_state_copy(RowCopy c, cudaStream_t s);

// Kernel attributes of the tensor-core kernels, set once per device (ops.cu).
cudaError_t ensure_tc_kernels(int* dev_out);

}  // namespace fr
