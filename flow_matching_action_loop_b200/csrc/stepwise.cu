// Stepwise kernels: one kernel per operation of the velocity, CUDA cores only.
//
// This is the simple kernel set of the library.  It runs the f32 workload
// (FFMA, no TF32), the FP8 calibration measure pass, and any handle created
// with FR_PATH_STEPWISE.  Activations are float32 buffers that already hold
// values on the projection-input grid (bf16-rounded, or e4m3 code values),
// so a GEMM multiplies exactly the operands the method defines.
//
// Operations (PhyAI page, optimisation paragraph; FlashRT walkthrough,
// component 8 for the memory-bound ones):
//   temb      time MLP of the sinusoidal embedding, once per load
//   inproj    h = W_in x + b_in + temb_k
//   rmsnorm_q a = Q(h / sqrt(mean h^2 + eps) * gamma)
//   gemm      C (+)= alpha * A W^T
//   rope_qkv  QKV split, RoPE at positions P..P+H-1, K/V into the KV cache
//   attention softmax(q K^T / sqrt(dh)) V over [prefix; actions]
//   gelu_mul  u = Q(gelu_tanh(gate) * up)
//   final     x += dt * (W_out bf16(RMSNorm(h)) + b_out)
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"

namespace fr {
namespace {

__device__ __forceinline__ float round_bf16(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

__device__ __forceinline__ float e4m3_value(float v) {
  __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
  __half_raw hr = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);
  return __half2float(__half(hr));
}

__device__ __forceinline__ void atomic_max_abs(unsigned* slot, float v) {
  atomicMax(slot, __float_as_uint(fabsf(v)));   // non-negative floats order like their bits
}

// Writes one projection input element according to the quantisation mode.
__device__ __forceinline__ float quantise(float v, int qmode, float inv_sa, unsigned* amax) {
  switch (qmode) {
    case Q_BF16: return round_bf16(v);
    case Q_E4M3: return e4m3_value(v * inv_sa);
    case Q_MEASURE: atomic_max_abs(amax, v); return v;
    default: return v;
  }
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  const int nw = (blockDim.x + 31) >> 5;
  for (int i = 0; i < nw; ++i) t += red[i];   // same order in every thread
  return t;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = -INFINITY;
  const int nw = (blockDim.x + 31) >> 5;
  for (int i = 0; i < nw; ++i) t = fmaxf(t, red[i]);
  return t;
}

// ------------------------------------------------------------------ time MLP (once per load)
__global__ void k_temb(const float* __restrict__ w_t1, const float* __restrict__ b_t1,
                       const float* __restrict__ w_t2, const float* __restrict__ b_t2,
                       float* __restrict__ temb, int D, int time_dim, int K, double time_base,
                       int rb) {
  extern __shared__ float sm[];
  float* e = sm;              // [time_dim]
  float* z = sm + time_dim;   // [D]
  const int k = blockIdx.x;
  const double t = 1.0 - static_cast<double>(k) / K;   // R1
  const int half = time_dim / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double w = pow(time_base, -static_cast<double>(i) / half);   // R2
    float s = static_cast<float>(sin(t * w)), c = static_cast<float>(cos(t * w));
    e[i] = rb ? round_bf16(s) : s;
    e[half + i] = rb ? round_bf16(c) : c;
  }
  __syncthreads();
  for (int n = threadIdx.x; n < D; n += blockDim.x) {
    const float* row = w_t1 + static_cast<size_t>(n) * time_dim;
    float acc = 0.f;
    for (int i = 0; i < time_dim; ++i) acc = fmaf(row[i], e[i], acc);
    acc += b_t1[n];
    const float sv = acc / (1.f + expf(-acc));
    z[n] = rb ? round_bf16(sv) : sv;
  }
  __syncthreads();
  for (int n = threadIdx.x; n < D; n += blockDim.x) {
    const float* row = w_t2 + static_cast<size_t>(n) * D;
    float acc = 0.f;
    for (int m = 0; m < D; ++m) acc = fmaf(row[m], z[m], acc);
    temb[static_cast<size_t>(k) * D + n] = acc + b_t2[n];
  }
}

// ------------------------------------------------------------------ in-proj + time
__global__ void k_inproj(const float* __restrict__ x, const float* __restrict__ w_in,
                         const float* __restrict__ b_in, const float* __restrict__ temb_k,
                         float* __restrict__ h, int D, int A, int rb) {
  extern __shared__ float xs[];
  const int t = blockIdx.x;
  for (int a = threadIdx.x; a < A; a += blockDim.x) {
    const float v = x[static_cast<size_t>(t) * A + a];
    xs[a] = rb ? round_bf16(v) : v;
  }
  __syncthreads();
  for (int n = threadIdx.x; n < D; n += blockDim.x) {
    const float* row = w_in + static_cast<size_t>(n) * A;
    float acc = 0.f;
    for (int a = 0; a < A; ++a) acc = fmaf(row[a], xs[a], acc);
    h[static_cast<size_t>(t) * D + n] = acc + b_in[n] + (temb_k ? temb_k[n] : 0.f);   // no temb: adaRMS
  }
}

// ------------------------------------------------------------------ RMSNorm + quantise
__global__ void k_rmsnorm_q(const float* __restrict__ h, const float* __restrict__ gamma,
                            float* __restrict__ out, int D, float eps, int qmode,
                            const float* __restrict__ s_a, unsigned* amax) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* row = h + static_cast<size_t>(t) * D;
  float ss = 0.f;
  for (int k = threadIdx.x; k < D; k += blockDim.x) ss = fmaf(row[k], row[k], ss);
  ss = block_sum(ss, red);
  const float r = 1.0f / sqrtf(ss / D + eps);
  const float inv_sa = (qmode == Q_E4M3) ? 1.0f / *s_a : 1.0f;
  for (int k = threadIdx.x; k < D; k += blockDim.x)
    out[static_cast<size_t>(t) * D + k] = quantise(row[k] * r * gamma[k], qmode, inv_sa, amax);
}

// ------------------------------------------------------------------ SIMT GEMM  C (+)= alpha A W^T
template <typename WT>
__device__ __forceinline__ float wload(const WT* p);
template <>
__device__ __forceinline__ float wload<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float wload<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <>
__device__ __forceinline__ float wload<uint8_t>(const uint8_t* p) {
  __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(*p), __NV_E4M3);
  return __half2float(__half(hr));
}

constexpr int GT = 64, GN = 64, GK = 16;

template <typename WT>
__global__ void __launch_bounds__(256) k_gemm(const float* __restrict__ A, int lda,
                                              const WT* __restrict__ W, const float* __restrict__ alpha,
                                              float* __restrict__ C, int ldc, int T, int N, int Kd,
                                              int accumulate, const float* __restrict__ bias,
                                              const float* __restrict__ gate) {
  __shared__ float As[GK][GT + 4];
  __shared__ float Ws[GK][GN + 4];
  const int t0 = blockIdx.y * GT, n0 = blockIdx.x * GN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < Kd; k0 += GK) {
    for (int i = threadIdx.x; i < GT * GK; i += blockDim.x) {
      const int r = i / GK, kk = i % GK;
      const int t = t0 + r, k = k0 + kk;
      As[kk][r] = (t < T && k < Kd) ? A[static_cast<size_t>(t) * lda + k] : 0.f;
      const int n = n0 + r;
      Ws[kk][r] = (n < N && k < Kd) ? wload<WT>(W + static_cast<size_t>(n) * Kd + k) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float al = alpha ? *alpha : 1.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float* c = C + static_cast<size_t>(t) * ldc + n;
      float v = al * acc[i][j];
      if (gate) v *= gate[n];   // adaRMS gated residual update
      if (bias) v += bias[n];   // adaRMS shift folded into the projection (W b)
      *c = accumulate ? *c + v : v;
    }
  }
}

// ------------------------------------------------------------------ KV cache element access
__device__ __forceinline__ float kv_get(const void* base, size_t idx, int bf) {
  return bf ? __bfloat162float(static_cast<const __nv_bfloat16*>(base)[idx])
            : static_cast<const float*>(base)[idx];
}
__device__ __forceinline__ void kv_put(void* base, size_t idx, float v, int bf) {
  if (bf) static_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else static_cast<float*>(base)[idx] = v;
}

// ------------------------------------------------------------------ QKV split + RoPE
// qkv [T][(Hq+2Hkv)dh] -> q [B][Hq][H][dh] (rotated), K/V cache slot P+i of this layer
// (cache layer slice [B_max][Hkv][S_max][dh]).
__global__ void k_rope_qkv(const float* __restrict__ qkv, float* __restrict__ q, void* kv_k,
                           void* kv_v, int kv_bf, const float* __restrict__ cos_t,
                           const float* __restrict__ sin_t, int H, int P, int S_max, int Hq,
                           int Hkv, int dh, int rb) {
  const int t = blockIdx.x;
  const int b = t / H, i = t % H;
  const int pos = P + i;
  const int half = dh / 2;
  const int nq = (Hq + 2 * Hkv) * dh;
  const float* row = qkv + static_cast<size_t>(t) * nq;
  const float* c = cos_t + static_cast<size_t>(pos) * half;
  const float* s = sin_t + static_cast<size_t>(pos) * half;
  // q and k heads: rotate-half
  for (int idx = threadIdx.x; idx < (Hq + Hkv) * half; idx += blockDim.x) {
    const int head = idx / half, d = idx % half;
    const float lo = row[head * dh + d], hi = row[head * dh + d + half];
    const float r0 = lo * c[d] - hi * s[d];
    const float r1 = lo * s[d] + hi * c[d];
    if (head < Hq) {
      float* qo = q + ((static_cast<size_t>(b) * Hq + head) * H + i) * dh;
      qo[d] = rb ? round_bf16(r0) : r0;
      qo[d + half] = rb ? round_bf16(r1) : r1;
    } else {
      const int g = head - Hq;
      const size_t base = ((static_cast<size_t>(b) * Hkv + g) * S_max + pos) * dh;
      kv_put(kv_k, base + d, r0, kv_bf);
      kv_put(kv_k, base + d + half, r1, kv_bf);
    }
  }
  for (int idx = threadIdx.x; idx < Hkv * dh; idx += blockDim.x) {
    const int g = idx / dh, d = idx % dh;
    const size_t base = ((static_cast<size_t>(b) * Hkv + g) * S_max + pos) * dh;
    kv_put(kv_v, base + d, row[(Hq + Hkv + g) * dh + d], kv_bf);
  }
}

// ------------------------------------------------------------------ prefix ingest
// in [L][B_src][P][Hkv][dh] (samples b0 .. b0+nb-1) -> cache [L][B_max][Hkv][S_max][dh] at the
// slots of `map`, K rotated at position p.
__global__ void k_prefix_ingest(const void* k_in, const void* v_in, void* kv_k, void* kv_v,
                                int kv_bf, const float* __restrict__ cos_t,
                                const float* __restrict__ sin_t, int B_src, int b0, int nb,
                                const __grid_constant__ SlotMap map, int B_max, int P,
                                int S_max, int Hkv, int dh, int rotate) {
  const long row = blockIdx.x;     // over L*nb*P*Hkv
  const int g = static_cast<int>(row % Hkv);
  const int p = static_cast<int>((row / Hkv) % P);
  const int bl = static_cast<int>((row / (static_cast<long>(Hkv) * P)) % nb);
  const int l = static_cast<int>(row / (static_cast<long>(Hkv) * P * nb));
  const int slot = map.n ? map.slot[bl] : b0 + bl;
  const size_t src = ((((static_cast<size_t>(l) * B_src + b0 + bl) * P + p) * Hkv) + g) * dh;
  const size_t dst = ((((static_cast<size_t>(l) * B_max + slot) * Hkv + g) * S_max) + p) * dh;
  const int half = dh / 2;
  for (int d = threadIdx.x; d < half; d += blockDim.x) {
    const float lo = kv_get(k_in, src + d, kv_bf), hi = kv_get(k_in, src + d + half, kv_bf);
    float r0 = lo, r1 = hi;
    if (rotate) {
      const float c = cos_t[static_cast<size_t>(p) * half + d], s = sin_t[static_cast<size_t>(p) * half + d];
      r0 = lo * c - hi * s;
      r1 = lo * s + hi * c;
    }
    kv_put(kv_k, dst + d, r0, kv_bf);
    kv_put(kv_k, dst + d + half, r1, kv_bf);
  }
  for (int d = threadIdx.x; d < dh; d += blockDim.x)
    kv_put(kv_v, dst + d, kv_get(v_in, src + d, kv_bf), kv_bf);
}

// ------------------------------------------------------------------ attention (one query row per block)
__global__ void k_attention(const float* __restrict__ q, const void* kv_k, const void* kv_v,
                            int kv_bf, float* __restrict__ act, int ld_act, int H, int P,
                            int S_max, int Hq, int Hkv, int dh, int qmode,
                            const float* __restrict__ s_a, unsigned* amax) {
  extern __shared__ float sm[];
  __shared__ float red[32];
  const int i = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const int g = (j * Hkv) / Hq;   // R7: consecutive query-head groups
  const int S = P + H;
  float* qs = sm;                 // [dh]
  float* p = sm + dh;             // [S]
  const float* qrow = q + ((static_cast<size_t>(b) * Hq + j) * H + i) * dh;
  for (int d = threadIdx.x; d < dh; d += blockDim.x) qs[d] = qrow[d];
  __syncthreads();
  const size_t kv0 = (static_cast<size_t>(b) * Hkv + g) * S_max * dh;
  const float scale = 1.0f / sqrtf(static_cast<float>(dh));
  float mx = -INFINITY;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    float acc = 0.f;
    for (int d = 0; d < dh; ++d) acc = fmaf(qs[d], kv_get(kv_k, kv0 + static_cast<size_t>(s) * dh + d, kv_bf), acc);
    acc *= scale;
    p[s] = acc;
    mx = fmaxf(mx, acc);
  }
  mx = block_max(mx, red);
  float sum = 0.f;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const float e = expf(p[s] - mx);
    p[s] = e;
    sum += e;
  }
  sum = block_sum(sum, red);
  const float inv = 1.0f / sum;
  const float inv_sa = (qmode == Q_E4M3) ? 1.0f / *s_a : 1.0f;
  float* out = act + (static_cast<size_t>(b) * H + i) * ld_act + static_cast<size_t>(j) * dh;
  for (int d = threadIdx.x; d < dh; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc = fmaf(p[s], kv_get(kv_v, kv0 + static_cast<size_t>(s) * dh + d, kv_bf), acc);
    out[d] = quantise(acc * inv, qmode, inv_sa, amax);
  }
}

// ------------------------------------------------------------------ GeLU(gate) * up
__global__ void k_gelu_mul(const float* __restrict__ gu, float* __restrict__ act, int T, int F,
                           int qmode, const float* __restrict__ s_a, unsigned* amax) {
  const size_t n = static_cast<size_t>(T) * F;
  const float inv_sa = (qmode == Q_E4M3) ? 1.0f / *s_a : 1.0f;
  const float c0 = 0.7978845608028654f;   // sqrt(2/pi)
  for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t t = idx / F, f = idx % F;
    const float g = gu[t * 2 * F + f], u = gu[t * 2 * F + F + f];
    const float ge = 0.5f * g * (1.f + tanhf(c0 * (g + 0.044715f * g * g * g)));
    act[t * F + f] = quantise(ge * u, qmode, inv_sa, amax);
  }
}

// ------------------------------------------------------------------ final norm + out-proj + Euler
__global__ void k_final(const float* __restrict__ h, const float* __restrict__ g_f,
                        const float* __restrict__ w_out, const float* __restrict__ b_out,
                        float* __restrict__ x, int D, int A, float eps, float dt, int rb) {
  extern __shared__ float hn[];
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* row = h + static_cast<size_t>(t) * D;
  float ss = 0.f;
  for (int k = threadIdx.x; k < D; k += blockDim.x) ss = fmaf(row[k], row[k], ss);
  ss = block_sum(ss, red);
  const float r = 1.0f / sqrtf(ss / D + eps);
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    const float v = row[k] * r * g_f[k];
    hn[k] = rb ? round_bf16(v) : v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int a = warp; a < A; a += nw) {
    const float* wr = w_out + static_cast<size_t>(a) * D;
    float acc = 0.f;
    for (int k = lane; k < D; k += 32) acc = fmaf(wr[k], hn[k], acc);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      float* xp = x + static_cast<size_t>(t) * A + a;
      *xp = *xp + dt * (acc + b_out[a]);
    }
  }
}

}  // namespace

// ------------------------------------------------------------------ launchers
void launch_temb(const float* w_t1, const float* b_t1, const float* w_t2, const float* b_t2,
                 float* temb, int D, int time_dim, int K, float time_base, int rb, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(time_dim + D) * sizeof(float);
  k_temb<<<K, 256, smem, s>>>(w_t1, b_t1, w_t2, b_t2, temb, D, time_dim, K, time_base, rb);
}

void launch_inproj(const float* x, const float* w_in, const float* b_in, const float* temb_k,
                   float* h, int T, int D, int A, int rb, cudaStream_t s) {
  k_inproj<<<T, 256, A * sizeof(float), s>>>(x, w_in, b_in, temb_k, h, D, A, rb);
}

void launch_rmsnorm_q(const float* h, const float* gamma, float* out, int T, int D, float eps,
                      int qmode, const float* s_a, unsigned* amax, cudaStream_t s) {
  k_rmsnorm_q<<<T, 256, 0, s>>>(h, gamma, out, D, eps, qmode, s_a, amax);
}

void launch_gemm(const float* A, int lda, const void* W, int wtype, const float* alpha, float* C,
                 int ldc, int T, int N, int Kd, int accumulate, cudaStream_t s, const float* bias,
                 const float* gate) {
  dim3 grid((N + GN - 1) / GN, (T + GT - 1) / GT);
  switch (wtype) {
    case W_F32:
      k_gemm<float><<<grid, 256, 0, s>>>(A, lda, static_cast<const float*>(W), alpha, C, ldc, T, N, Kd, accumulate,
                                         bias, gate);
      break;
    case W_BF16:
      k_gemm<__nv_bfloat16><<<grid, 256, 0, s>>>(A, lda, static_cast<const __nv_bfloat16*>(W), alpha, C, ldc, T, N,
                                                 Kd, accumulate, bias, gate);
      break;
    default:
      k_gemm<uint8_t><<<grid, 256, 0, s>>>(A, lda, static_cast<const uint8_t*>(W), alpha, C, ldc, T, N, Kd,
                                           accumulate, bias, gate);
      break;
  }
}

// ------------------------------------------------------------------ adaRMS preparation (load time)
// out[r][j] = in[r * in_ld + j], rounded to bf16 when rb
__global__ void k_round_rows(const float* __restrict__ in, int in_ld, float* __restrict__ out, int rows, int n,
                             int rb) {
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < static_cast<long>(rows) * n;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const float v = in[(i / n) * in_ld + i % n];
    out[i] = rb ? round_bf16(v) : v;
  }
}

// out[r][j] = 1 + in[r * in_ld + j]: the norm gain 1 + s of each modulation row
__global__ void k_one_plus(const float* __restrict__ in, int in_ld, float* __restrict__ out, int rows, int n) {
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < static_cast<long>(rows) * n;
       i += static_cast<long>(gridDim.x) * blockDim.x)
    out[i] = 1.0f + in[(i / n) * in_ld + i % n];
}

void launch_round_rows(const float* in, int in_ld, float* out, int rows, int n, int rb, cudaStream_t s) {
  k_round_rows<<<148, 256, 0, s>>>(in, in_ld, out, rows, n, rb);
}

void launch_one_plus(const float* in, int in_ld, float* out, int rows, int n, cudaStream_t s) {
  k_one_plus<<<148, 256, 0, s>>>(in, in_ld, out, rows, n);
}

void launch_rope_qkv(const float* qkv, float* q, void* kv_k, void* kv_v, int kv_bf,
                     const float* cos_t, const float* sin_t, int B, int H, int P, int S_max, int Hq,
                     int Hkv, int dh, int rb, cudaStream_t s) {
  k_rope_qkv<<<B * H, 128, 0, s>>>(qkv, q, kv_k, kv_v, kv_bf, cos_t, sin_t, H, P, S_max, Hq, Hkv, dh, rb);
}

void launch_prefix_ingest(const void* k_in, const void* v_in, void* kv_k, void* kv_v, int kv_bf,
                          const float* cos_t, const float* sin_t, int L, int B_src, int b0, int nb,
                          const SlotMap& map, int B_max, int P, int S_max, int Hkv, int dh, int rotate,
                          cudaStream_t s) {
  const long rows = static_cast<long>(L) * nb * P * Hkv;
  k_prefix_ingest<<<static_cast<unsigned>(rows), 64, 0, s>>>(k_in, v_in, kv_k, kv_v, kv_bf, cos_t, sin_t,
                                                             B_src, b0, nb, map, B_max, P, S_max, Hkv, dh,
                                                             rotate);
}

void launch_attention(const float* q, const void* kv_k, const void* kv_v, int kv_bf, float* act,
                      int ld_act, int B, int H, int P, int S_max, int Hq, int Hkv, int dh, int qmode,
                      const float* s_a, unsigned* amax, cudaStream_t s) {
  dim3 grid(H, Hq, B);
  const size_t smem = static_cast<size_t>(dh + P + H) * sizeof(float);
  k_attention<<<grid, 128, smem, s>>>(q, kv_k, kv_v, kv_bf, act, ld_act, H, P, S_max, Hq, Hkv, dh,
                                      qmode, s_a, amax);
}

void launch_gelu_mul(const float* gu, float* act, int T, int F, int qmode, const float* s_a,
                     unsigned* amax, cudaStream_t s) {
  const size_t n = static_cast<size_t>(T) * F;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  k_gelu_mul<<<blocks, 256, 0, s>>>(gu, act, T, F, qmode, s_a, amax);
}

void launch_final(const float* h, const float* g_f, const float* w_out, const float* b_out, float* x,
                  int T, int D, int A, float eps, float dt, int rb, cudaStream_t s) {
  k_final<<<T, 256, D * sizeof(float), s>>>(h, g_f, w_out, b_out, x, D, A, eps, dt, rb);
}

}  // namespace fr
