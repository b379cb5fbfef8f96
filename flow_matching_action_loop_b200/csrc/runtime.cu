// Runtime of the action-expert library: the handle, the weight packer and the
// C ABI declared in fr.h.
//
// Design points taken from the pages (prior art, re-planned for one B200):
//   - FlashRT walkthrough, "exec/: C ABI execution contract": named device
//     buffers are the only state; cold start is separate from the hot call.
//   - FlashRT walkthrough, component 7: the hot call takes pointers only and
//     allocates nothing -- here every buffer is carved out of one allocation in
//     fr_create.
//   - APXInf page, section "一次跑得快，还要持续跑得稳": fixed execution path,
//     memory allocated up front.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <cmath>
#include <vector>

#include "internal.h"
#include "tc_kernels.h"
#include "tensor_path.h"

namespace fr {

static thread_local char g_err[1024] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

int cuda_fail(cudaError_t e, const char* what) {
  set_error("CUDA error %d (%s) in %s", static_cast<int>(e), cudaGetErrorString(e), what);
  return FR_ERR_CUDA;
}

}  // namespace fr

using namespace fr;

struct fr_handle {
  fr_config cfg{};
  int device = 0;
  int S_max = 0;            // P_max + H KV slots per (layer, sample, kv head)
  int n_qkv = 0, dq = 0;    // (Hq+2Hkv)dh, Hq dh
  int wtype = W_F32;
  size_t welem = 4;
  int kv_bf = 0;
  int path = FR_PATH_STEPWISE;
  bool weights_loaded = false;
  bool scales_set = false;
  int prefix_B = 0, prefix_P = 0;

  char* pool = nullptr;
  size_t pool_bytes = 0;

  std::vector<StepwiseWeights> lw;
  float *w_in = nullptr, *b_in = nullptr, *w_out = nullptr, *b_out = nullptr;
  float *w_t1 = nullptr, *b_t1 = nullptr, *w_t2 = nullptr, *b_t2 = nullptr, *g_f = nullptr;
  float* temb = nullptr;                    // [K][D]
  float *rope_cos = nullptr, *rope_sin = nullptr;   // [S_max][dh/2]
  char *kv_k = nullptr, *kv_v = nullptr;    // [L][B_max][Hkv][S_max][dh]
  size_t kv_layer_bytes = 0;
  float *x = nullptr, *h = nullptr, *act = nullptr, *qkv = nullptr, *q = nullptr, *gu = nullptr;
  float *s_a = nullptr, *s_w = nullptr, *alpha = nullptr;   // [L][4]
  unsigned* amax = nullptr;                 // [L][4]
  unsigned* status = nullptr;
  std::vector<float> h_sw, h_sa;

  TensorPath* tp = nullptr;                 // tensor-core kernel set (bf16/fp8)

  // adaptive RMSNorm (cfg.adarms): every step's norm modulation, precomputed by fr_load_weights
  float* ada_stage = nullptr;   // one modulation weight [3D][D] and its bias [3D], staged for the GEMM
  float* ada_c = nullptr;       // [K][D] condition of each step: the time embedding, rounded like an input
  float* ada_mod = nullptr;     // [K][L][2][3D] (scale | shift | gate) of the pre-attention / pre-MLP norm
  float* ada_gain = nullptr;    // [K][L][2][D] 1 + scale
  float* ada_modf = nullptr;    // [K][2D] final norm (scale | shift)
  float* ada_gainf = nullptr;   // [K][D]
  float* ada_bout = nullptr;    // [K][A] b_out + W_out shift_f
  float* ada_cq = nullptr;      // [K][L][(Hq+2Hkv)dh] W_qkv shift_1
  float* ada_cg = nullptr;      // [K][L][2F] W_gu shift_2
};

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Carver {
  size_t off = 0;
  template <typename T>
  size_t take(size_t count, size_t align = 256) {
    off = align_up(off, align);
    const size_t o = off;
    off += count * sizeof(T);
    return o;
  }
};

int validate(const fr_config& c) {
  if (c.L < 1 || c.D < 1 || c.Hq < 1 || c.Hkv < 1 || c.dh < 2 || c.F < 1 || c.H < 1 || c.A < 1 ||
      c.B_max < 1 || c.P_max < 1 || c.K < 1 || c.time_dim < 2) {
    set_error("fr_create: every size must be positive");
    return FR_ERR_ARG;
  }
  if (c.dtype < FR_DTYPE_F32 || c.dtype > FR_DTYPE_W4A16 || c.path < FR_PATH_AUTO || c.path > FR_PATH_TENSOR) {
    set_error("fr_create: bad dtype/path enum");
    return FR_ERR_ARG;
  }
  // RMSNorm's eps, RoPE's theta and the time embedding's base: finite, and positive where a power is taken
  if (!std::isfinite(c.eps) || c.eps < 0.f || !std::isfinite(c.rope_theta) || c.rope_theta <= 0.f ||
      !std::isfinite(c.time_base) || c.time_base <= 0.f) {
    set_error("fr_create: need eps >= 0, rope_theta > 0 and time_base > 0, all finite");
    return FR_ERR_ARG;
  }
  if ((c.dh & 1) || (c.time_dim & 1) || (c.Hq % c.Hkv)) {
    set_error("fr_create: dh and time_dim must be even and Hq a multiple of Hkv");
    return FR_ERR_UNSUPPORTED;
  }
  if (c.A > 4096 || c.D > 16384 || c.time_dim > 4096 || c.P_max + c.H > 16384) {
    set_error("fr_create: A <= 4096, D <= 16384, time_dim <= 4096, P_max+H <= 16384");
    return FR_ERR_UNSUPPORTED;
  }
  if (c.path == FR_PATH_TENSOR && c.dtype == FR_DTYPE_F32) {
    set_error("fr_create: the tensor-core path needs a bf16, fp8 or w4a16 handle");
    return FR_ERR_UNSUPPORTED;
  }
  if (c.role != FR_ROLE_EXPERT && c.role != FR_ROLE_PREFIX) {
    set_error("fr_create: bad role enum");
    return FR_ERR_ARG;
  }
  if (c.role == FR_ROLE_PREFIX &&
      ((c.dtype != FR_DTYPE_BF16 && c.dtype != FR_DTYPE_W4A16) || c.path == FR_PATH_STEPWISE || c.adarms)) {
    set_error("fr_create: the prefix pass runs bf16 or w4a16 on the tensor-core path, without adarms");
    return FR_ERR_UNSUPPORTED;
  }
  return FR_OK;
}

int qmode_of(const fr_handle* h, bool measure) {
  if (h->cfg.dtype == FR_DTYPE_F32) return Q_NONE;
  if (h->cfg.dtype == FR_DTYPE_BF16 || h->cfg.dtype == FR_DTYPE_W4A16) return Q_BF16;
  return measure ? Q_MEASURE : Q_E4M3;
}

// Stepwise loop over all K steps for B samples (x already holds x0).
void run_stepwise(fr_handle* h, int B, bool measure, cudaStream_t s) {
  const fr_config& c = h->cfg;
  const int T = B * c.H;
  const int rb = c.dtype != FR_DTYPE_F32;
  const int qm = qmode_of(h, measure);
  const float dt = static_cast<float>(-1.0 / c.K);
  const int P = h->prefix_P;
  const bool ada = c.adarms != 0;
  for (int k = 0; k < c.K; ++k) {
    // adaptive RMSNorm: the time embedding conditions the norms instead of being added
    launch_inproj(h->x, h->w_in, h->b_in, ada ? nullptr : h->temb + static_cast<size_t>(k) * c.D, h->h, T, c.D,
                  c.A, rb, s);
    for (int l = 0; l < c.L; ++l) {
      const StepwiseWeights& w = h->lw[l];
      const size_t kl = static_cast<size_t>(k) * c.L + l;
      const float* gain1 = ada ? h->ada_gain + kl * 2 * c.D : w.g1;
      const float* gain2 = ada ? gain1 + c.D : w.g2;
      const float* gate1 = ada ? h->ada_mod + kl * 6 * c.D + 2 * c.D : nullptr;
      const float* gate2 = ada ? gate1 + 3 * c.D : nullptr;
      const float* bias_qkv = ada ? h->ada_cq + kl * h->n_qkv : nullptr;
      const float* bias_gu = ada ? h->ada_cg + kl * 2 * c.F : nullptr;
      void* kk = h->kv_k + l * h->kv_layer_bytes;
      void* vv = h->kv_v + l * h->kv_layer_bytes;
      const float* sa = h->s_a + l * PI_COUNT;
      unsigned* am = h->amax + l * PI_COUNT;
      auto alpha = [&](int i) -> const float* {
        if (c.dtype != FR_DTYPE_FP8) return nullptr;
        return (measure ? h->s_w : h->alpha) + l * PI_COUNT + i;
      };
      launch_rmsnorm_q(h->h, gain1, h->act, T, c.D, c.eps, qm, sa + PI_QKV, am + PI_QKV, s);
      launch_gemm(h->act, c.D, w.wqkv, h->wtype, alpha(PI_QKV), h->qkv, h->n_qkv, T, h->n_qkv, c.D, 0, s,
                  bias_qkv);
      launch_rope_qkv(h->qkv, h->q, kk, vv, h->kv_bf, h->rope_cos, h->rope_sin, B, c.H, P, h->S_max,
                      c.Hq, c.Hkv, c.dh, rb, s);
      launch_attention(h->q, kk, vv, h->kv_bf, h->act, h->dq, B, c.H, P, h->S_max, c.Hq, c.Hkv, c.dh,
                       qm, sa + PI_O, am + PI_O, s);
      launch_gemm(h->act, h->dq, w.wo, h->wtype, alpha(PI_O), h->h, c.D, T, c.D, h->dq, 1, s, nullptr, gate1);
      launch_rmsnorm_q(h->h, gain2, h->act, T, c.D, c.eps, qm, sa + PI_GU, am + PI_GU, s);
      launch_gemm(h->act, c.D, w.wgu, h->wtype, alpha(PI_GU), h->gu, 2 * c.F, T, 2 * c.F, c.D, 0, s, bias_gu);
      launch_gelu_mul(h->gu, h->act, T, c.F, qm, sa + PI_DOWN, am + PI_DOWN, s);
      launch_gemm(h->act, c.F, w.wd, h->wtype, alpha(PI_DOWN), h->h, c.D, T, c.D, c.F, 1, s, nullptr, gate2);
    }
    launch_final(h->h, ada ? h->ada_gainf + static_cast<size_t>(k) * c.D : h->g_f, h->w_out,
                 ada ? h->ada_bout + static_cast<size_t>(k) * c.A : h->b_out, h->x, T, c.D, c.A, c.eps, dt, rb, s);
  }
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return FR_OK;
}

// Host packing helpers --------------------------------------------------------------
void pack_rows(std::vector<uint8_t>& dst, size_t& off, const float* src, size_t n, int wtype, double scale) {
  if (wtype == W_F32) {
    std::memcpy(dst.data() + off, src, n * 4);
    off += n * 4;
  } else if (wtype == W_BF16) {
    fr_round_bf16(src, reinterpret_cast<uint16_t*>(dst.data() + off), n);
    off += n * 2;
  } else {
    fr_quantize_e4m3(src, dst.data() + off, n, scale);
    off += n;
  }
}

// w4a16: the 4-bit codes and scales of a [rows][cols] weight, then bf16(q * s) per element
// (q * s is exact in float32: 3 magnitude bits times an 8-bit significand).
void pack_w4_dequant(std::vector<uint8_t>& dst, size_t& off, const float* src, int rows, int cols) {
  const int ng = (cols + FR_W4_GROUP - 1) / FR_W4_GROUP;
  std::vector<int8_t> q(static_cast<size_t>(rows) * cols);
  std::vector<uint16_t> sb(static_cast<size_t>(rows) * ng);
  fr_quantize_w4(src, rows, cols, q.data(), sb.data());
  std::vector<float> deq(q.size());
  for (int r = 0; r < rows; ++r)
    for (int c = 0; c < cols; ++c) {
      const uint32_t u = static_cast<uint32_t>(sb[static_cast<size_t>(r) * ng + c / FR_W4_GROUP]) << 16;
      float sv;
      std::memcpy(&sv, &u, 4);
      deq[static_cast<size_t>(r) * cols + c] = static_cast<float>(q[static_cast<size_t>(r) * cols + c]) * sv;
    }
  fr_round_bf16(deq.data(), reinterpret_cast<uint16_t*>(dst.data() + off), deq.size());
  off += deq.size() * 2;
}

std::vector<float> rounded_f32(const float* src, size_t n, bool to_bf16) {
  std::vector<float> out(src, src + n);
  if (to_bf16) {
    std::vector<uint16_t> b(n);
    fr_round_bf16(src, b.data(), n);
    for (size_t i = 0; i < n; ++i) {
      const uint32_t u = static_cast<uint32_t>(b[i]) << 16;
      std::memcpy(&out[i], &u, 4);
    }
  }
  return out;
}

float max_abs(const float* p, size_t n) {
  float m = 0.f;
  for (size_t i = 0; i < n; ++i) m = std::max(m, std::fabs(p[i]));
  return m;
}

}  // namespace

extern "C" {

const char* fr_last_error(void) { return g_err; }

int fr_create(const fr_config* cfg, int device, fr_handle** out) {
  if (!cfg || !out) {
    set_error("fr_create: NULL argument");
    return FR_ERR_ARG;
  }
  *out = nullptr;
  int rc = validate(*cfg);
  if (rc) return rc;
  FR_CUDA(cudaSetDevice(device));
  fr_handle* h = new fr_handle();
  h->cfg = *cfg;
  h->device = device;
  const fr_config& c = h->cfg;
  h->S_max = c.P_max + c.H;
  h->n_qkv = (c.Hq + 2 * c.Hkv) * c.dh;
  h->dq = c.Hq * c.dh;
  // w4a16: the stepwise kernels read the dequantised operand bf16(q * s)
  h->wtype = c.dtype == FR_DTYPE_F32 ? W_F32 : (c.dtype == FR_DTYPE_FP8 ? W_E4M3 : W_BF16);
  h->welem = c.dtype == FR_DTYPE_F32 ? 4 : (c.dtype == FR_DTYPE_FP8 ? 1 : 2);
  h->kv_bf = c.dtype != FR_DTYPE_F32;
  h->path = c.path;
  if (h->path == FR_PATH_AUTO) h->path = (c.dtype == FR_DTYPE_F32) ? FR_PATH_STEPWISE : FR_PATH_TENSOR;
  if (h->path == FR_PATH_TENSOR && !tensor_path_supports(c)) {
    if (c.path == FR_PATH_TENSOR || c.role == FR_ROLE_PREFIX) {
      set_error("fr_create: sizes outside the tensor-core path (%s)", tensor_path_limits());
      delete h;
      return FR_ERR_UNSUPPORTED;
    }
    h->path = FR_PATH_STEPWISE;
  }

  const size_t T_max = static_cast<size_t>(c.B_max) * c.H;
  const size_t D = c.D, F = c.F;
  const size_t w_layer = (static_cast<size_t>(h->n_qkv) * D + D * h->dq + 2 * F * D + D * F);
  const size_t act_w = std::max({D, F, static_cast<size_t>(h->dq)});
  Carver cv;
  std::vector<size_t> lw_off(c.L);
  for (int l = 0; l < c.L; ++l) lw_off[l] = cv.take<uint8_t>(w_layer * h->welem);
  const size_t o_gain = cv.take<float>(2 * D * c.L);
  const size_t o_w_in = cv.take<float>(D * c.A), o_b_in = cv.take<float>(D);
  const size_t o_w_out = cv.take<float>(c.A * D), o_b_out = cv.take<float>(c.A);
  const size_t o_w_t1 = cv.take<float>(D * c.time_dim), o_b_t1 = cv.take<float>(D);
  const size_t o_w_t2 = cv.take<float>(D * D), o_b_t2 = cv.take<float>(D), o_g_f = cv.take<float>(D);
  const size_t o_temb = cv.take<float>(static_cast<size_t>(c.K) * D);
  const size_t half = c.dh / 2;
  const size_t o_cos = cv.take<float>(h->S_max * half), o_sin = cv.take<float>(h->S_max * half);
  h->kv_layer_bytes = align_up(static_cast<size_t>(c.B_max) * c.Hkv * h->S_max * c.dh * (h->kv_bf ? 2 : 4), 256);
  const size_t o_kvk = cv.take<uint8_t>(h->kv_layer_bytes * c.L), o_kvv = cv.take<uint8_t>(h->kv_layer_bytes * c.L);
  const size_t o_x = cv.take<float>(T_max * c.A), o_h = cv.take<float>(T_max * D);
  const size_t o_act = cv.take<float>(T_max * act_w), o_qkv = cv.take<float>(T_max * h->n_qkv);
  const size_t o_q = cv.take<float>(T_max * h->dq), o_gu = cv.take<float>(T_max * 2 * F);
  const size_t o_sa = cv.take<float>(c.L * PI_COUNT), o_sw = cv.take<float>(c.L * PI_COUNT);
  const size_t o_alpha = cv.take<float>(c.L * PI_COUNT), o_amax = cv.take<unsigned>(c.L * PI_COUNT);
  const size_t o_status = cv.take<unsigned>(4);
  const bool ada = c.adarms != 0;
  const size_t KL = static_cast<size_t>(c.K) * c.L;
  const size_t o_ada_stage = cv.take<float>(ada ? 3 * D * (D + 1) : 0);
  const size_t o_ada_c = cv.take<float>(ada ? c.K * D : 0);
  const size_t o_ada_mod = cv.take<float>(ada ? KL * 6 * D : 0);
  const size_t o_ada_gain = cv.take<float>(ada ? KL * 2 * D : 0);
  const size_t o_ada_modf = cv.take<float>(ada ? c.K * 2 * D : 0);
  const size_t o_ada_gainf = cv.take<float>(ada ? c.K * D : 0);
  const size_t o_ada_bout = cv.take<float>(ada ? static_cast<size_t>(c.K) * c.A : 0);
  const size_t o_ada_cq = cv.take<float>(ada ? KL * h->n_qkv : 0);
  const size_t o_ada_cg = cv.take<float>(ada ? KL * 2 * F : 0);
  size_t tp_bytes = 0;
  if (h->path == FR_PATH_TENSOR) tp_bytes = tensor_path_bytes(c);
  const size_t o_tp = cv.take<uint8_t>(tp_bytes, 1024);
  h->pool_bytes = align_up(cv.off, 1024);

  cudaError_t e = cudaMalloc(&h->pool, h->pool_bytes);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e, "cudaMalloc(handle pool)");
  }
  e = cudaMemset(h->pool, 0, h->pool_bytes);
  if (e != cudaSuccess) {
    cudaFree(h->pool);
    delete h;
    return cuda_fail(e, "cudaMemset(handle pool)");
  }
  char* p = h->pool;
  h->lw.resize(c.L);
  for (int l = 0; l < c.L; ++l) {
    char* base = p + lw_off[l];
    StepwiseWeights& w = h->lw[l];
    w.wqkv = base;
    w.wo = base + static_cast<size_t>(h->n_qkv) * D * h->welem;
    w.wgu = static_cast<const char*>(w.wo) + D * h->dq * h->welem;
    w.wd = static_cast<const char*>(w.wgu) + 2 * F * D * h->welem;
    w.g1 = reinterpret_cast<float*>(p + o_gain) + 2 * D * l;
    w.g2 = w.g1 + D;
  }
  h->w_in = reinterpret_cast<float*>(p + o_w_in);
  h->b_in = reinterpret_cast<float*>(p + o_b_in);
  h->w_out = reinterpret_cast<float*>(p + o_w_out);
  h->b_out = reinterpret_cast<float*>(p + o_b_out);
  h->w_t1 = reinterpret_cast<float*>(p + o_w_t1);
  h->b_t1 = reinterpret_cast<float*>(p + o_b_t1);
  h->w_t2 = reinterpret_cast<float*>(p + o_w_t2);
  h->b_t2 = reinterpret_cast<float*>(p + o_b_t2);
  h->g_f = reinterpret_cast<float*>(p + o_g_f);
  h->temb = reinterpret_cast<float*>(p + o_temb);
  h->rope_cos = reinterpret_cast<float*>(p + o_cos);
  h->rope_sin = reinterpret_cast<float*>(p + o_sin);
  h->kv_k = p + o_kvk;
  h->kv_v = p + o_kvv;
  h->x = reinterpret_cast<float*>(p + o_x);
  h->h = reinterpret_cast<float*>(p + o_h);
  h->act = reinterpret_cast<float*>(p + o_act);
  h->qkv = reinterpret_cast<float*>(p + o_qkv);
  h->q = reinterpret_cast<float*>(p + o_q);
  h->gu = reinterpret_cast<float*>(p + o_gu);
  h->s_a = reinterpret_cast<float*>(p + o_sa);
  h->s_w = reinterpret_cast<float*>(p + o_sw);
  h->alpha = reinterpret_cast<float*>(p + o_alpha);
  h->amax = reinterpret_cast<unsigned*>(p + o_amax);
  h->status = reinterpret_cast<unsigned*>(p + o_status);
  if (ada) {
    h->ada_stage = reinterpret_cast<float*>(p + o_ada_stage);
    h->ada_c = reinterpret_cast<float*>(p + o_ada_c);
    h->ada_mod = reinterpret_cast<float*>(p + o_ada_mod);
    h->ada_gain = reinterpret_cast<float*>(p + o_ada_gain);
    h->ada_modf = reinterpret_cast<float*>(p + o_ada_modf);
    h->ada_gainf = reinterpret_cast<float*>(p + o_ada_gainf);
    h->ada_bout = reinterpret_cast<float*>(p + o_ada_bout);
    h->ada_cq = reinterpret_cast<float*>(p + o_ada_cq);
    h->ada_cg = reinterpret_cast<float*>(p + o_ada_cg);
  }

  // RoPE tables (R6): float64 math on the host, rounded once to float32.
  std::vector<float> ct(h->S_max * half), st(h->S_max * half);
  fr_rope_tables(h->S_max, c.dh, c.rope_theta, ct.data(), st.data());
  e = cudaMemcpy(h->rope_cos, ct.data(), ct.size() * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->rope_sin, st.data(), st.size() * 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    fr_destroy(h);
    return cuda_fail(e, "cudaMemcpy(rope tables)");
  }
  if (h->path == FR_PATH_TENSOR) {
    TensorPathBuffers tb{};
    tb.base = p + o_tp;
    tb.bytes = tp_bytes;
    tb.rope_cos = h->rope_cos;
    tb.rope_sin = h->rope_sin;
    tb.kv_k = h->kv_k;
    tb.kv_v = h->kv_v;
    tb.kv_layer_bytes = h->kv_layer_bytes;
    tb.x = h->x;
    tb.temb = h->temb;
    tb.w_in = h->w_in;
    tb.b_in = h->b_in;
    tb.w_out = h->w_out;
    tb.b_out = h->b_out;
    tb.g_f = h->g_f;
    tb.alpha = h->alpha;
    tb.s_a = h->s_a;
    tb.status = h->status;
    tb.ada_gain = h->ada_gain;
    tb.ada_mod = h->ada_mod;
    tb.ada_gainf = h->ada_gainf;
    tb.ada_bout = h->ada_bout;
    tb.ada_cq = h->ada_cq;
    tb.ada_cg = h->ada_cg;
    rc = tensor_path_create(c, tb, &h->tp);
    if (rc) {
      fr_destroy(h);
      return rc;
    }
  }
  *out = h;
  return FR_OK;
}

// Adaptive RMSNorm, once per weight load: the condition of every Euler step (its time embedding,
// rounded like a projection input), each norm's (scale | shift | gate) = W_mod c + b_mod, the gains
// 1 + scale, and the shifts folded into the projections they feed: W_qkv shift_1, W_gu shift_2 and
// b_out + W_out shift_f.  Runs the stepwise GEMM kernel on the stored (rounded / quantised) weights.
int prepare_adarms(fr_handle* h, const fr_weights& w, bool rb, cudaStream_t s) {
  const fr_config& c = h->cfg;
  const int D = c.D, K = c.K, L = c.L;
  const int ld_mod = L * 6 * D;   // row stride of ada_mod between steps
  launch_round_rows(h->temb, D, h->ada_c, K, D, rb ? 1 : 0, s);
  auto modulate = [&](const float* W, const float* b, int rows, float* out, int ldo) -> int {
    std::vector<float> v = rounded_f32(W, static_cast<size_t>(rows) * D, rb);
    FR_CUDA(cudaMemcpyAsync(h->ada_stage, v.data(), v.size() * 4, cudaMemcpyHostToDevice, s));
    FR_CUDA(cudaMemcpyAsync(h->ada_stage + v.size(), b, static_cast<size_t>(rows) * 4, cudaMemcpyHostToDevice, s));
    launch_gemm(h->ada_c, D, h->ada_stage, W_F32, nullptr, out, ldo, K, rows, D, 0, s, h->ada_stage + v.size());
    int rc = check_launch("adaRMS modulation GEMM");
    if (rc) return rc;
    FR_CUDA(cudaStreamSynchronize(s));   // the stage is rewritten by the next call
    return FR_OK;
  };
  int rc;
  for (int l = 0; l < L; ++l) {
    const fr_layer_weights& lw = w.layers[l];
    if ((rc = modulate(lw.w_mod1, lw.b_mod1, 3 * D, h->ada_mod + static_cast<size_t>(l) * 6 * D, ld_mod))) return rc;
    if ((rc = modulate(lw.w_mod2, lw.b_mod2, 3 * D, h->ada_mod + static_cast<size_t>(l) * 6 * D + 3 * D, ld_mod)))
      return rc;
  }
  if ((rc = modulate(w.w_modf, w.b_modf, 2 * D, h->ada_modf, 2 * D))) return rc;
  launch_one_plus(h->ada_mod, 3 * D, h->ada_gain, K * L * 2, D, s);
  launch_one_plus(h->ada_modf, 2 * D, h->ada_gainf, K, D, s);
  const bool fp8 = c.dtype == FR_DTYPE_FP8;
  for (int l = 0; l < L; ++l) {   // shifts folded into the projections (fp8: dequantised by s_w)
    const StepwiseWeights& lw = h->lw[l];
    const float* shift1 = h->ada_mod + static_cast<size_t>(l) * 6 * D + D;
    const float* shift2 = shift1 + 3 * D;
    launch_gemm(shift1, ld_mod, lw.wqkv, h->wtype, fp8 ? h->s_w + l * PI_COUNT + PI_QKV : nullptr,
                h->ada_cq + static_cast<size_t>(l) * h->n_qkv, L * h->n_qkv, K, h->n_qkv, D, 0, s);
    launch_gemm(shift2, ld_mod, lw.wgu, h->wtype, fp8 ? h->s_w + l * PI_COUNT + PI_GU : nullptr,
                h->ada_cg + static_cast<size_t>(l) * 2 * c.F, L * 2 * c.F, K, 2 * c.F, D, 0, s);
  }
  launch_gemm(h->ada_modf + D, 2 * D, h->w_out, W_F32, nullptr, h->ada_bout, c.A, K, c.A, D, 0, s, h->b_out);
  return check_launch("adaRMS preparation kernels");
}

int fr_load_weights(fr_handle* h, const fr_weights* w_in, fr_stream_t stream) {
  if (!h || !w_in || !w_in->layers) {
    set_error("fr_load_weights: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (c.role != FR_ROLE_PREFIX && (!w_in->w_in || !w_in->b_in || !w_in->w_out || !w_in->b_out || !w_in->w_t1 ||
                                   !w_in->b_t1 || !w_in->w_t2 || !w_in->b_t2)) {
    set_error("fr_load_weights: NULL argument");
    return FR_ERR_ARG;
  }
  const bool ada = c.adarms != 0;
  const bool pre = c.role == FR_ROLE_PREFIX;   // the backbone: only the layer tensors are read
  if (!pre && (ada ? (!w_in->w_modf || !w_in->b_modf) : !w_in->g_f)) {
    set_error(ada ? "fr_load_weights: adarms handle without w_modf / b_modf" : "fr_load_weights: NULL g_f");
    return FR_ERR_ARG;
  }
  for (int l = 0; l < c.L; ++l) {
    const fr_layer_weights& L = w_in->layers[l];
    if (!L.wq || !L.wk || !L.wv || !L.wo || !L.wg || !L.wu || !L.wd ||
        (ada ? (!L.w_mod1 || !L.b_mod1 || !L.w_mod2 || !L.b_mod2) : (!L.g1 || !L.g2))) {
      set_error("fr_load_weights: NULL tensor in layer %d", l);
      return FR_ERR_ARG;
    }
  }
  // adaptive RMSNorm replaces the static gains: they are unused, read as ones
  const std::vector<float> ones(ada ? static_cast<size_t>(c.D) : 0, 1.f);
  std::vector<fr_layer_weights> layers(w_in->layers, w_in->layers + c.L);
  fr_weights wcopy = *w_in;
  if (ada) {
    for (fr_layer_weights& L : layers) L.g1 = L.g2 = ones.data();
    wcopy.g_f = ones.data();
  }
  wcopy.layers = layers.data();
  const fr_weights* w = &wcopy;
  FR_CUDA(cudaSetDevice(h->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t D = c.D, F = c.F, dq = h->dq, nkv = static_cast<size_t>(c.Hkv) * c.dh;
  const bool rb = c.dtype != FR_DTYPE_F32;
  h->h_sw.assign(static_cast<size_t>(c.L) * PI_COUNT, 1.f);
  std::vector<uint8_t> buf;
  std::vector<float> gains(2 * D * c.L);
  for (int l = 0; l < c.L; ++l) {
    const fr_layer_weights& L = w->layers[l];
    const size_t bytes = (static_cast<size_t>(h->n_qkv) * D + D * dq + 2 * F * D + D * F) * h->welem;
    buf.assign(bytes, 0);
    size_t off = 0;
    double sw[PI_COUNT] = {1, 1, 1, 1};
    if (c.dtype == FR_DTYPE_FP8) {   // one scale per fused projection: s_w = max|w| / 448 (R11)
      sw[PI_QKV] = std::max({max_abs(L.wq, dq * D), max_abs(L.wk, nkv * D), max_abs(L.wv, nkv * D)}) / 448.0;
      sw[PI_O] = max_abs(L.wo, D * dq) / 448.0;
      sw[PI_GU] = std::max(max_abs(L.wg, F * D), max_abs(L.wu, F * D)) / 448.0;
      sw[PI_DOWN] = max_abs(L.wd, D * F) / 448.0;
      for (int i = 0; i < PI_COUNT; ++i) {
        if (!(sw[i] > 0)) sw[i] = 1.0;   // an all-zero tensor quantises to zero codes with any scale
        h->h_sw[l * PI_COUNT + i] = static_cast<float>(sw[i]);
      }
    }
    if (c.dtype == FR_DTYPE_W4A16) {
      const int iD = c.D, iF = c.F, idq = static_cast<int>(dq), inkv = static_cast<int>(nkv);
      pack_w4_dequant(buf, off, L.wq, idq, iD);
      pack_w4_dequant(buf, off, L.wk, inkv, iD);
      pack_w4_dequant(buf, off, L.wv, inkv, iD);
      pack_w4_dequant(buf, off, L.wo, iD, idq);
      pack_w4_dequant(buf, off, L.wg, iF, iD);
      pack_w4_dequant(buf, off, L.wu, iF, iD);
      pack_w4_dequant(buf, off, L.wd, iD, iF);
    } else {
      pack_rows(buf, off, L.wq, dq * D, h->wtype, sw[PI_QKV]);
      pack_rows(buf, off, L.wk, nkv * D, h->wtype, sw[PI_QKV]);
      pack_rows(buf, off, L.wv, nkv * D, h->wtype, sw[PI_QKV]);
      pack_rows(buf, off, L.wo, D * dq, h->wtype, sw[PI_O]);
      pack_rows(buf, off, L.wg, F * D, h->wtype, sw[PI_GU]);
      pack_rows(buf, off, L.wu, F * D, h->wtype, sw[PI_GU]);
      pack_rows(buf, off, L.wd, D * F, h->wtype, sw[PI_DOWN]);
    }
    FR_CUDA(cudaMemcpy(const_cast<void*>(h->lw[l].wqkv), buf.data(), bytes, cudaMemcpyHostToDevice));
    std::memcpy(&gains[2 * D * l], L.g1, D * 4);
    std::memcpy(&gains[2 * D * l + D], L.g2, D * 4);
    if (h->tp) {
      int rc = tensor_path_pack_layer(h->tp, l, L, sw);
      if (rc) return rc;
    }
  }
  FR_CUDA(cudaMemcpy(const_cast<float*>(h->lw[0].g1), gains.data(), gains.size() * 4, cudaMemcpyHostToDevice));
  auto up = [&](float* dst, const float* src, size_t n, bool round) -> int {
    std::vector<float> v = rounded_f32(src, n, round);
    FR_CUDA(cudaMemcpy(dst, v.data(), n * 4, cudaMemcpyHostToDevice));
    return FR_OK;
  };
  int rc = FR_OK;
  FR_CUDA(cudaMemcpy(h->s_w, h->h_sw.data(), h->h_sw.size() * 4, cudaMemcpyHostToDevice));
  if (!pre) {   // in/out-proj, time MLP and final norm of the expert
    if ((rc = up(h->w_in, w->w_in, D * c.A, rb))) return rc;
    if ((rc = up(h->b_in, w->b_in, D, false))) return rc;
    if ((rc = up(h->w_out, w->w_out, c.A * D, rb))) return rc;
    if ((rc = up(h->b_out, w->b_out, c.A, false))) return rc;
    if ((rc = up(h->w_t1, w->w_t1, D * c.time_dim, rb))) return rc;
    if ((rc = up(h->b_t1, w->b_t1, D, false))) return rc;
    if ((rc = up(h->w_t2, w->w_t2, D * D, rb))) return rc;
    if ((rc = up(h->b_t2, w->b_t2, D, false))) return rc;
    if ((rc = up(h->g_f, w->g_f, D, false))) return rc;
    launch_temb(h->w_t1, h->b_t1, h->w_t2, h->b_t2, h->temb, c.D, c.time_dim, c.K, c.time_base, rb, s);
    if ((rc = check_launch("time MLP kernel"))) return rc;
    if (ada && (rc = prepare_adarms(h, *w, rb, s))) return rc;
  }
  FR_CUDA(cudaStreamSynchronize(s));
  if (h->tp) {
    rc = tensor_path_finish_load(h->tp, s);
    if (rc) return rc;
  }
  h->weights_loaded = true;
  h->scales_set = false;
  return FR_OK;
}

int fr_set_prefix_kv(fr_handle* h, const void* k_dev, const void* v_dev, int B, int P, unsigned flags,
                     fr_stream_t stream) {
  if (!h || !k_dev || !v_dev) {
    set_error("fr_set_prefix_kv: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (B < 1 || B > c.B_max || P < 1 || P > c.P_max) {
    set_error("fr_set_prefix_kv: need 1 <= B <= %d and 1 <= P <= %d (got B=%d P=%d)", c.B_max, c.P_max, B, P);
    return FR_ERR_SHAPE;
  }
  if (flags & ~FR_PREFIX_K_ROTATED) {
    set_error("fr_set_prefix_kv: unknown flag bits 0x%x", flags);
    return FR_ERR_ARG;
  }
  if (c.role != FR_ROLE_EXPERT) {
    set_error("fr_set_prefix_kv: a prefix-pass handle writes its KV with fr_prefill");
    return FR_ERR_STATE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int rotate = (flags & FR_PREFIX_K_ROTATED) ? 0 : 1;
  SlotMap identity{};
  launch_prefix_ingest(k_dev, v_dev, h->kv_k, h->kv_v, h->kv_bf, h->rope_cos, h->rope_sin, c.L, B, 0, B, identity,
                       c.B_max, P, h->S_max, c.Hkv, c.dh, rotate, s);
  int rc = check_launch("prefix ingest kernel");
  if (rc) return rc;
  h->prefix_B = B;
  h->prefix_P = P;
  return FR_OK;
}

// ------------------------------------------------------------------ execution contract across chunks

int fr_refresh_prefix_kv(fr_handle* h, const void* k_dev, const void* v_dev, const int* slots, int n, int P,
                         unsigned flags, fr_stream_t stream) {
  if (!h || !k_dev || !v_dev || !slots || n < 1) {
    set_error("fr_refresh_prefix_kv: NULL argument or n < 1");
    return FR_ERR_ARG;
  }
  if (flags & ~FR_PREFIX_K_ROTATED) {
    set_error("fr_refresh_prefix_kv: unknown flag bits 0x%x", flags);
    return FR_ERR_ARG;
  }
  if (h->prefix_B < 1) {
    set_error("fr_refresh_prefix_kv: no prefix set (call fr_set_prefix_kv or fr_capsule_restore first)");
    return FR_ERR_STATE;
  }
  if (P != h->prefix_P) {
    set_error("fr_refresh_prefix_kv: P=%d differs from the cached prefix length %d", P, h->prefix_P);
    return FR_ERR_SHAPE;
  }
  std::vector<char> seen(h->prefix_B, 0);
  for (int i = 0; i < n; ++i) {
    if (slots[i] < 0 || slots[i] >= h->prefix_B) {
      set_error("fr_refresh_prefix_kv: slot %d outside the %d cached samples", slots[i], h->prefix_B);
      return FR_ERR_SHAPE;
    }
    if (seen[slots[i]]) {
      set_error("fr_refresh_prefix_kv: slot %d given twice", slots[i]);
      return FR_ERR_ARG;
    }
    seen[slots[i]] = 1;
  }
  const fr_config& c = h->cfg;
  FR_CUDA(cudaSetDevice(h->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int rotate = (flags & FR_PREFIX_K_ROTATED) ? 0 : 1;
  for (int b0 = 0; b0 < n; b0 += SLOT_MAP_MAX) {
    SlotMap m{};
    m.n = std::min(SLOT_MAP_MAX, n - b0);
    for (int i = 0; i < m.n; ++i) m.slot[i] = slots[b0 + i];
    launch_prefix_ingest(k_dev, v_dev, h->kv_k, h->kv_v, h->kv_bf, h->rope_cos, h->rope_sin, c.L, n, b0, m.n, m,
                         c.B_max, P, h->S_max, c.Hkv, c.dh, rotate, s);
    int rc = check_launch("prefix ingest kernel");
    if (rc) return rc;
  }
  return FR_OK;
}

int fr_get_buffer(const fr_handle* h, const char* name, void** dev, size_t* bytes) {
  if (!h || !name || !dev || !bytes) {
    set_error("fr_get_buffer: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  const size_t rope = static_cast<size_t>(h->S_max) * (c.dh / 2) * sizeof(float);
  struct Named {
    const char* name;
    void* p;
    size_t n;
  };
  const Named table[] = {
      {"kv_k", h->kv_k, h->kv_layer_bytes * c.L},
      {"kv_v", h->kv_v, h->kv_layer_bytes * c.L},
      {"rope_cos", h->rope_cos, rope},
      {"rope_sin", h->rope_sin, rope},
      {"temb", h->temb, static_cast<size_t>(c.K) * c.D * sizeof(float)},
      {"s_act", h->s_a, static_cast<size_t>(c.L) * PI_COUNT * sizeof(float)},
      {"status", h->status, sizeof(unsigned)},
  };
  for (const Named& e : table)
    if (std::strcmp(e.name, name) == 0) {
      *dev = e.p;
      *bytes = e.n;
      return FR_OK;
    }
  set_error("fr_get_buffer: no buffer named '%s'", name);
  return FR_ERR_ARG;
}

namespace {

struct CapsuleLayout {
  size_t kv_bytes = 0;   // one of K or V: [L][B][Hkv][P][dh]
  size_t v_off = 0, x_off = 0, total = 0;
};

CapsuleLayout capsule_layout(const fr_config& c, int B, int P, int with_x) {
  CapsuleLayout l;
  const size_t elem = c.dtype == FR_DTYPE_F32 ? 4 : 2;
  l.kv_bytes = static_cast<size_t>(c.L) * B * c.Hkv * P * c.dh * elem;
  l.v_off = align_up(l.kv_bytes, 256);
  l.x_off = l.v_off + align_up(l.kv_bytes, 256);
  l.total = l.x_off + (with_x ? align_up(static_cast<size_t>(B) * c.H * c.A * sizeof(float), 256) : 0);
  return l;
}

// Rows of the prefix KV between the handle's cache and a capsule's [L][B][Hkv][P][dh] layout.
// to_capsule: cache slot map[b] -> capsule sample b; otherwise capsule sample map[b] -> slot b.
int copy_prefix(const fr_handle* h, char* cap, int B_cap, int P, const int* map, int n, bool to_capsule,
                cudaStream_t s) {
  const fr_config& c = h->cfg;
  const long long rowb = static_cast<long long>(c.dh) * (h->kv_bf ? 2 : 4);
  const CapsuleLayout lay = capsule_layout(c, B_cap, P, 0);
  const long long cache[4] = {static_cast<long long>(h->kv_layer_bytes), c.Hkv * h->S_max * rowb, h->S_max * rowb, rowb};
  const long long capsule[4] = {static_cast<long long>(B_cap) * c.Hkv * P * rowb, c.Hkv * P * rowb, P * rowb, rowb};
  const long long* src = to_capsule ? cache : capsule;
  const long long* dst = to_capsule ? capsule : cache;
  char* cache_k = h->kv_k;
  char* cache_v = h->kv_v;
  char* cap_k = cap;
  char* cap_v = cap + lay.v_off;
  for (int b0 = 0; b0 < n; b0 += SLOT_MAP_MAX) {
    RowCopy rc{};
    rc.parts = 2;
    rc.src[0] = to_capsule ? cache_k : cap_k;
    rc.src[1] = to_capsule ? cache_v : cap_v;
    rc.dst[0] = (to_capsule ? cap_k : cache_k) + b0 * dst[1];
    rc.dst[1] = (to_capsule ? cap_v : cache_v) + b0 * dst[1];
    rc.n_outer = c.L;
    rc.n_sample = std::min(SLOT_MAP_MAX, n - b0);
    rc.n_mid = c.Hkv;
    rc.n_row = P;
    rc.s_outer = src[0], rc.s_sample = src[1], rc.s_mid = src[2], rc.s_row = src[3];
    rc.d_outer = dst[0], rc.d_sample = dst[1], rc.d_mid = dst[2], rc.d_row = dst[3];
    rc.row_bytes = rowb;
    for (int i = 0; i < rc.n_sample; ++i) rc.map[i] = map[b0 + i];
    launch_state_copy(rc, s);
    int r = check_launch("state copy kernel");
    if (r) return r;
  }
  return FR_OK;
}

// x [B][H][A] float32 rows: dst sample b <- src sample map[b].
int copy_x(const fr_config& c, const float* src, float* dst, const int* map, int n, cudaStream_t s) {
  const long long xb = static_cast<long long>(c.H) * c.A * sizeof(float);
  for (int b0 = 0; b0 < n; b0 += SLOT_MAP_MAX) {
    RowCopy rc{};
    rc.parts = 1;
    rc.src[0] = reinterpret_cast<const char*>(src);
    rc.dst[0] = reinterpret_cast<char*>(dst) + b0 * xb;
    rc.n_outer = rc.n_mid = rc.n_row = 1;
    rc.n_sample = std::min(SLOT_MAP_MAX, n - b0);
    rc.s_sample = rc.d_sample = xb;
    rc.row_bytes = xb;
    for (int i = 0; i < rc.n_sample; ++i) rc.map[i] = map[b0 + i];
    launch_state_copy(rc, s);
    int r = check_launch("state copy kernel");
    if (r) return r;
  }
  return FR_OK;
}

}  // namespace

size_t fr_capsule_bytes(const fr_config* cfg, int B, int P, int with_x) {
  if (!cfg || validate(*cfg) != FR_OK || B < 1 || B > cfg->B_max || P < 1 || P > cfg->P_max) return 0;
  return capsule_layout(*cfg, B, P, with_x ? 1 : 0).total;
}

int fr_capsule_save(const fr_handle* h, void* cap_dev, size_t cap_bytes, int B, const float* x_dev,
                    fr_capsule* desc, fr_stream_t stream) {
  if (!h || !cap_dev || !desc) {
    set_error("fr_capsule_save: NULL argument");
    return FR_ERR_ARG;
  }
  if (h->prefix_B < 1) {
    set_error("fr_capsule_save: no prefix set");
    return FR_ERR_STATE;
  }
  if (B < 1 || B > h->prefix_B) {
    set_error("fr_capsule_save: need 1 <= B <= %d cached samples (got %d)", h->prefix_B, B);
    return FR_ERR_SHAPE;
  }
  const fr_config& c = h->cfg;
  const int P = h->prefix_P;
  const CapsuleLayout lay = capsule_layout(c, B, P, x_dev != nullptr);
  if (cap_bytes < lay.total) {
    set_error("fr_capsule_save: capsule buffer of %zu bytes, %zu needed", cap_bytes, lay.total);
    return FR_ERR_SHAPE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::vector<int> identity(B);
  for (int b = 0; b < B; ++b) identity[b] = b;
  char* cap = static_cast<char*>(cap_dev);
  int rc = copy_prefix(h, cap, B, P, identity.data(), B, true, s);
  if (rc) return rc;
  if (x_dev) {
    rc = copy_x(c, x_dev, reinterpret_cast<float*>(cap + lay.x_off), identity.data(), B, s);
    if (rc) return rc;
  }
  fr_capsule d{};
  d.magic = FR_CAPSULE_MAGIC;
  d.L = c.L, d.Hkv = c.Hkv, d.dh = c.dh, d.kv_bytes_per_elem = h->kv_bf ? 2 : 4;
  d.H = c.H, d.A = c.A;
  d.B = B, d.P = P;
  d.has_x = x_dev != nullptr;
  d.bytes = lay.total;
  *desc = d;
  return FR_OK;
}

int fr_capsule_restore(fr_handle* h, const void* cap_dev, const fr_capsule* desc, const int* map, int B,
                       float* x_dev, fr_stream_t stream) {
  if (!h || !cap_dev || !desc) {
    set_error("fr_capsule_restore: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (c.role != FR_ROLE_EXPERT) {
    set_error("fr_capsule_restore: not an expert handle");
    return FR_ERR_STATE;
  }
  if (desc->magic != FR_CAPSULE_MAGIC || desc->B < 1 || desc->P < 1) {
    set_error("fr_capsule_restore: not a capsule description (magic 0x%x, B=%d, P=%d)", desc->magic, desc->B,
              desc->P);
    return FR_ERR_ARG;
  }
  if (desc->L != c.L || desc->Hkv != c.Hkv || desc->dh != c.dh || desc->kv_bytes_per_elem != (h->kv_bf ? 2 : 4) ||
      desc->H != c.H || desc->A != c.A) {
    set_error("fr_capsule_restore: capsule written by a handle of another shape");
    return FR_ERR_SHAPE;
  }
  if (B < 1 || B > c.B_max || desc->P > c.P_max) {
    set_error("fr_capsule_restore: need 1 <= B <= %d and P <= %d (got B=%d, capsule P=%d)", c.B_max, c.P_max, B,
              desc->P);
    return FR_ERR_SHAPE;
  }
  std::vector<int> m(B);
  for (int b = 0; b < B; ++b) {
    m[b] = map ? map[b] : b;
    if (m[b] < 0 || m[b] >= desc->B) {
      if (!map) {
        set_error("fr_capsule_restore: B=%d without a map, the capsule holds %d samples", B, desc->B);
        return FR_ERR_SHAPE;
      }
      set_error("fr_capsule_restore: map[%d]=%d outside the capsule's %d samples", b, m[b], desc->B);
      return FR_ERR_ARG;
    }
  }
  if (x_dev && !desc->has_x) {
    set_error("fr_capsule_restore: x requested but the capsule holds none");
    return FR_ERR_STATE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* cap = const_cast<char*>(static_cast<const char*>(cap_dev));   // read only
  int rc = copy_prefix(h, cap, desc->B, desc->P, m.data(), B, false, s);
  if (rc) return rc;
  if (x_dev) {
    const CapsuleLayout lay = capsule_layout(c, desc->B, desc->P, 1);
    rc = copy_x(c, reinterpret_cast<const float*>(cap + lay.x_off), x_dev, m.data(), B, s);
    if (rc) return rc;
  }
  h->prefix_B = B;
  h->prefix_P = desc->P;
  return FR_OK;
}

int fr_set_graph_capacity(fr_handle* h, int capacity) {
  if (!h || capacity < 1) {
    set_error("fr_set_graph_capacity: NULL handle or capacity < 1");
    return FR_ERR_ARG;
  }
  if (h->tp) {
    FR_CUDA(cudaSetDevice(h->device));   // evicted graphs are destroyed on the handle's device
    return tensor_path_set_graph_capacity(h->tp, capacity);
  }
  return FR_OK;
}

int fr_graph_count(const fr_handle* h) {
  if (!h) {
    set_error("fr_graph_count: NULL handle");
    return FR_ERR_ARG;
  }
  return h->tp ? tensor_path_graph_count(h->tp) : 0;
}

int fr_prefill(fr_handle* bb, const void* emb_dev, int B, int P, fr_handle* ex, fr_stream_t stream) {
  if (!bb || !emb_dev) {
    set_error("fr_prefill: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = bb->cfg;
  if (c.role != FR_ROLE_PREFIX || !bb->tp) {
    set_error("fr_prefill: not a prefix-pass handle (create it with role FR_ROLE_PREFIX)");
    return FR_ERR_STATE;
  }
  if (!bb->weights_loaded) {
    set_error("fr_prefill: no weights loaded");
    return FR_ERR_STATE;
  }
  if (B < 1 || B > c.B_max || P < 1 || P > c.H) {
    set_error("fr_prefill: need 1 <= B <= %d and 1 <= P <= %d (got B=%d P=%d)", c.B_max, c.H, B, P);
    return FR_ERR_SHAPE;
  }
  if (ex) {
    const fr_config& e = ex->cfg;
    if (e.role != FR_ROLE_EXPERT) {
      set_error("fr_prefill: the destination is not an expert handle");
      return FR_ERR_STATE;
    }
    if (ex->device != bb->device) {   // the copy kernel runs on the pass's device and writes the expert's cache
      set_error("fr_prefill: the expert handle is on device %d, the prefix pass on device %d", ex->device, bb->device);
      return FR_ERR_ARG;
    }
    if (e.L != c.L || e.Hkv != c.Hkv || e.dh != c.dh || !ex->kv_bf || B > e.B_max || P > e.P_max) {
      set_error("fr_prefill: expert KV [L=%d Hkv=%d dh=%d, B_max=%d P_max=%d, %s] cannot take the pass's "
                "[L=%d Hkv=%d dh=%d] for B=%d P=%d",
                e.L, e.Hkv, e.dh, e.B_max, e.P_max, ex->kv_bf ? "bf16" : "f32", c.L, c.Hkv, c.dh, B, P);
      return FR_ERR_SHAPE;
    }
  }
  FR_CUDA(cudaSetDevice(bb->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int rc = tensor_path_prefill(bb->tp, emb_dev, B, P, s);
  if (rc) return rc;
  if ((rc = check_launch("prefix pass"))) return rc;
  if (ex) {   // rows 0..P-1 of slots 0..B-1, every layer and KV head, into the expert's cache
    const long long rowb = static_cast<long long>(c.dh) * 2;
    for (int b0 = 0; b0 < B; b0 += SLOT_MAP_MAX) {
      RowCopy rcp{};
      rcp.parts = 2;
      rcp.n_outer = c.L;
      rcp.n_sample = std::min(SLOT_MAP_MAX, B - b0);
      rcp.n_mid = c.Hkv;
      rcp.n_row = P;
      rcp.s_outer = static_cast<long long>(bb->kv_layer_bytes);
      rcp.s_sample = c.Hkv * bb->S_max * rowb;
      rcp.s_mid = bb->S_max * rowb;
      rcp.s_row = rowb;
      rcp.d_outer = static_cast<long long>(ex->kv_layer_bytes);
      rcp.d_sample = ex->cfg.Hkv * ex->S_max * rowb;
      rcp.d_mid = ex->S_max * rowb;
      rcp.d_row = rowb;
      rcp.src[0] = bb->kv_k;
      rcp.src[1] = bb->kv_v;
      rcp.dst[0] = ex->kv_k + b0 * rcp.d_sample;
      rcp.dst[1] = ex->kv_v + b0 * rcp.d_sample;
      rcp.row_bytes = rowb;
      for (int i = 0; i < rcp.n_sample; ++i) rcp.map[i] = b0 + i;
      launch_state_copy(rcp, s);
      if ((rc = check_launch("state copy kernel"))) return rc;
    }
    ex->prefix_B = B;
    ex->prefix_P = P;
  }
  return FR_OK;
}

int fr_denoise(fr_handle* h, const float* x0_dev, float* x_out_dev, int B, fr_stream_t stream) {
  if (!h || !x0_dev || !x_out_dev) {
    set_error("fr_denoise: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (c.role != FR_ROLE_EXPERT) {
    set_error("fr_denoise: a prefix-pass handle runs fr_prefill, not the loop");
    return FR_ERR_STATE;
  }
  if (B < 1 || B > c.B_max) {
    set_error("fr_denoise: need 1 <= B <= %d (got %d)", c.B_max, B);
    return FR_ERR_SHAPE;
  }
  if (!h->weights_loaded) {
    set_error("fr_denoise: no weights loaded");
    return FR_ERR_STATE;
  }
  if (h->prefix_B < B) {
    set_error("fr_denoise: prefix KV set for %d samples, denoise asked for %d", h->prefix_B, B);
    return FR_ERR_STATE;
  }
  if (c.dtype == FR_DTYPE_FP8 && !h->scales_set) {
    set_error("fr_denoise: fp8 handle without activation scales (run fr_calibrate or fr_set_scales)");
    return FR_ERR_STATE;
  }
  FR_CUDA(cudaSetDevice(h->device));   // the handle's buffers, graphs and kernels live there
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t xbytes = static_cast<size_t>(B) * c.H * c.A * sizeof(float);
  if (h->path == FR_PATH_TENSOR) {
    int rc = tensor_path_denoise(h->tp, x0_dev, x_out_dev, B, h->prefix_P, s);
    if (rc) return rc;
    return check_launch("tensor path");
  }
  FR_CUDA(cudaMemcpyAsync(h->x, x0_dev, xbytes, cudaMemcpyDeviceToDevice, s));
  run_stepwise(h, B, false, s);
  FR_CUDA(cudaMemcpyAsync(x_out_dev, h->x, xbytes, cudaMemcpyDeviceToDevice, s));
  return check_launch("stepwise kernels");
}

int fr_calibrate(fr_handle* h, const float* x0_dev, const void* pk_dev, const void* pv_dev, int B, int P,
                 fr_stream_t stream) {
  if (!h || !x0_dev || !pk_dev || !pv_dev) {
    set_error("fr_calibrate: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (c.dtype != FR_DTYPE_FP8) {
    set_error("fr_calibrate: only fp8 handles are calibrated");
    return FR_ERR_STATE;
  }
  if (!h->weights_loaded) {
    set_error("fr_calibrate: no weights loaded");
    return FR_ERR_STATE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  int rc = fr_set_prefix_kv(h, pk_dev, pv_dev, B, P, 0, stream);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FR_CUDA(cudaMemsetAsync(h->amax, 0, c.L * PI_COUNT * sizeof(unsigned), s));
  FR_CUDA(cudaMemcpyAsync(h->x, x0_dev, static_cast<size_t>(B) * c.H * c.A * 4, cudaMemcpyDeviceToDevice, s));
  run_stepwise(h, B, true, s);
  if ((rc = check_launch("calibration kernels"))) return rc;
  std::vector<unsigned> am(c.L * PI_COUNT);
  FR_CUDA(cudaMemcpyAsync(am.data(), h->amax, am.size() * 4, cudaMemcpyDeviceToHost, s));
  FR_CUDA(cudaStreamSynchronize(s));
  std::vector<float> sa(am.size());
  for (size_t i = 0; i < am.size(); ++i) {
    float a;
    std::memcpy(&a, &am[i], 4);
    sa[i] = a > 0.f ? a / 448.0f : 1.0f;
  }
  return fr_set_scales(h, sa.data(), static_cast<int>(sa.size()));
}

int fr_get_scales(const fr_handle* h, float* s_act, float* s_w, int n) {
  if (!h || !s_act) {
    set_error("fr_get_scales: NULL argument");
    return FR_ERR_ARG;
  }
  if (h->cfg.dtype != FR_DTYPE_FP8 || !h->scales_set) {
    set_error("fr_get_scales: not an fp8 handle or scales not set");
    return FR_ERR_STATE;
  }
  if (n != h->cfg.L * PI_COUNT) {
    set_error("fr_get_scales: n must be L*4 = %d", h->cfg.L * PI_COUNT);
    return FR_ERR_SHAPE;
  }
  std::memcpy(s_act, h->h_sa.data(), n * 4);
  if (s_w) std::memcpy(s_w, h->h_sw.data(), n * 4);
  return FR_OK;
}

int fr_set_scales(fr_handle* h, const float* s_act, int n) {
  if (!h || !s_act) {
    set_error("fr_set_scales: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (c.dtype != FR_DTYPE_FP8 || !h->weights_loaded) {
    set_error("fr_set_scales: needs an fp8 handle with weights loaded");
    return FR_ERR_STATE;
  }
  if (n != c.L * PI_COUNT) {
    set_error("fr_set_scales: n must be L*4 = %d", c.L * PI_COUNT);
    return FR_ERR_SHAPE;
  }
  for (int i = 0; i < n; ++i) {
    if (!(s_act[i] > 0.f) || !std::isfinite(s_act[i])) {
      set_error("fr_set_scales: scale %d is not a positive finite number", i);
      return FR_ERR_ARG;
    }
  }
  FR_CUDA(cudaSetDevice(h->device));
  h->h_sa.assign(s_act, s_act + n);
  std::vector<float> alpha(n);
  for (int i = 0; i < n; ++i) alpha[i] = h->h_sa[i] * h->h_sw[i];   // alpha = act_scale x weight_scale
  FR_CUDA(cudaMemcpy(h->s_a, h->h_sa.data(), n * 4, cudaMemcpyHostToDevice));
  FR_CUDA(cudaMemcpy(h->alpha, alpha.data(), n * 4, cudaMemcpyHostToDevice));
  if (h->tp) {
    int rc = tensor_path_set_scales(h->tp, h->h_sa.data(), alpha.data());
    if (rc) return rc;
  }
  h->scales_set = true;
  return FR_OK;
}

int fr_selftest_wait(fr_handle* h, uint64_t limit_ns, fr_stream_t stream) {
  if (!h || limit_ns < 1000 || limit_ns > 100000000ull) {
    set_error("fr_selftest_wait: NULL handle or limit outside [1 us, 100 ms]");
    return FR_ERR_ARG;
  }
  FR_CUDA(cudaSetDevice(h->device));
  FR_CUDA(tc::launch_wait_selftest(h->status, static_cast<unsigned long long>(limit_ns),
                                   reinterpret_cast<cudaStream_t>(stream)));
  return FR_OK;
}

int fr_sync_status(fr_handle* h, fr_stream_t stream) {
  if (!h) {
    set_error("fr_sync_status: NULL handle");
    return FR_ERR_ARG;
  }
  FR_CUDA(cudaSetDevice(h->device));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned st[4] = {0, 0, 0, 0};
  FR_CUDA(cudaMemcpyAsync(st, h->status, sizeof(st), cudaMemcpyDeviceToHost, s));
  FR_CUDA(cudaStreamSynchronize(s));
  FR_CUDA(cudaMemsetAsync(h->status, 0, sizeof(st), s));
  FR_CUDA(cudaStreamSynchronize(s));
  if (st[0] & ST_TIMEOUT) {
    set_error("device wait gave up (phase word 0x%08x, block %u)", st[1], st[2]);
    return FR_ERR_TIMEOUT;
  }
  if (st[0] & ST_BOUNDS) {
    set_error("device bounds check failed (where 0x%08x, index %u)", st[1], st[2]);
    return FR_ERR_DEVICE;
  }
  return FR_OK;
}

void fr_destroy(fr_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  if (h->tp) tensor_path_destroy(h->tp);
  if (h->pool) cudaFree(h->pool);
  delete h;
}

int fr_read_kv(const fr_handle* h, int layer, int b, void* k_host, void* v_host, int n_slots) {
  if (!h || !k_host || !v_host) {
    set_error("fr_read_kv: NULL argument");
    return FR_ERR_ARG;
  }
  const fr_config& c = h->cfg;
  if (layer < 0 || layer >= c.L || b < 0 || b >= c.B_max || n_slots < 1 || n_slots > h->S_max) {
    set_error("fr_read_kv: index out of range");
    return FR_ERR_SHAPE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  FR_CUDA(cudaDeviceSynchronize());
  const size_t el = h->kv_bf ? 2 : 4;
  const size_t row = static_cast<size_t>(c.dh) * el;
  for (int g = 0; g < c.Hkv; ++g) {
    const size_t src = layer * h->kv_layer_bytes + ((static_cast<size_t>(b) * c.Hkv + g) * h->S_max) * row;
    const size_t dst = static_cast<size_t>(g) * n_slots * row;
    FR_CUDA(cudaMemcpy(static_cast<char*>(k_host) + dst, h->kv_k + src, n_slots * row, cudaMemcpyDeviceToHost));
    FR_CUDA(cudaMemcpy(static_cast<char*>(v_host) + dst, h->kv_v + src, n_slots * row, cudaMemcpyDeviceToHost));
  }
  return FR_OK;
}

int fr_get_rope_tables(const fr_handle* h, float* cos_host, float* sin_host, int n_pos) {
  if (!h || !cos_host || !sin_host) {
    set_error("fr_get_rope_tables: NULL argument");
    return FR_ERR_ARG;
  }
  if (n_pos < 1 || n_pos > h->S_max) {
    set_error("fr_get_rope_tables: n_pos must be in [1, %d]", h->S_max);
    return FR_ERR_SHAPE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  const size_t n = static_cast<size_t>(n_pos) * (h->cfg.dh / 2) * 4;
  FR_CUDA(cudaMemcpy(cos_host, h->rope_cos, n, cudaMemcpyDeviceToHost));
  FR_CUDA(cudaMemcpy(sin_host, h->rope_sin, n, cudaMemcpyDeviceToHost));
  return FR_OK;
}

const char* fr_path_name(const fr_handle* h) {
  if (!h) return "";
  return h->path == FR_PATH_TENSOR ? "tensor" : "stepwise";
}

int fr_launches_per_call(const fr_handle* h, int B) {
  if (!h) return 0;
  if (h->path == FR_PATH_TENSOR) return tensor_path_launches(h->tp, B, h->prefix_P > 0 ? h->prefix_P : h->cfg.P_max);
  return h->cfg.K * (2 + 9 * h->cfg.L);
}

int fr_set_exec_mode(fr_handle* h, int mode) {
  if (!h || mode < FR_EXEC_AUTO || mode > FR_EXEC_PERSISTENT) {
    set_error("fr_set_exec_mode: NULL handle or unknown mode");
    return FR_ERR_ARG;
  }
  if (h->path != FR_PATH_TENSOR || h->cfg.role != FR_ROLE_EXPERT) {
    set_error("fr_set_exec_mode: the handle does not run the tensor-core loop");
    return FR_ERR_STATE;
  }
  return tensor_path_set_exec_mode(h->tp, mode);
}

int fr_exec_mode(const fr_handle* h, int B) {
  if (!h) {
    set_error("fr_exec_mode: NULL handle");
    return FR_ERR_ARG;
  }
  if (h->path != FR_PATH_TENSOR) {
    set_error("fr_exec_mode: the handle does not run the tensor-core path");
    return FR_ERR_STATE;
  }
  cudaSetDevice(h->device);
  return tensor_path_exec(h->tp, B, h->prefix_P > 0 ? h->prefix_P : h->cfg.P_max);
}

int fr_device_checks(void) {
#ifdef FR_DEVICE_CHECKS
  return 1;
#else
  return 0;
#endif
}

int fr_debug_plan(const fr_config* cfg, int B, int P, int nsm, int max_dyn, int max_dyn2, int* out, int n_out) {
  if (!cfg || !out || n_out < 0 || nsm < 1 || max_dyn < 1 || max_dyn2 < 0) {
    set_error("fr_debug_plan: NULL or non-positive argument");
    return FR_ERR_ARG;
  }
  int rc = validate(*cfg);
  if (rc) return rc;
  if (!tensor_path_supports(*cfg)) {
    set_error("fr_debug_plan: the configuration is outside the tensor-core path (%s)", tensor_path_limits());
    return FR_ERR_UNSUPPORTED;
  }
  const int p_max = cfg->role == FR_ROLE_PREFIX ? cfg->H : cfg->P_max;
  if (B < 1 || B > cfg->B_max || P < 1 || P > p_max) {
    set_error("fr_debug_plan: B must be in [1, B_max] and P in [1, %d]", p_max);
    return FR_ERR_SHAPE;
  }
  return tensor_path_debug_plan(*cfg, B, P, nsm, max_dyn, max_dyn2, out, n_out);
}

int fr_debug_limit_extent(fr_handle* h, const char* buffer, uint64_t elems) {
  if (!h || !buffer) {
    set_error("fr_debug_limit_extent: NULL argument");
    return FR_ERR_ARG;
  }
  if (!fr_device_checks()) {
    set_error("fr_debug_limit_extent: this library was built without device bounds checks");
    return FR_ERR_UNSUPPORTED;
  }
  if (h->path != FR_PATH_TENSOR) {
    set_error("fr_debug_limit_extent: the handle does not run the tensor-core path");
    return FR_ERR_STATE;
  }
  FR_CUDA(cudaSetDevice(h->device));
  return tensor_path_limit_extent(h->tp, buffer, elems);
}

int fr_set_wait_limit(fr_handle* h, uint64_t limit_ns) {
  if (!h || limit_ns > 10000000000ull) {
    set_error("fr_set_wait_limit: NULL handle or limit above 10 s");
    return FR_ERR_ARG;
  }
  if (h->path == FR_PATH_TENSOR) tensor_path_set_wait_limit(h->tp, limit_ns);
  return FR_OK;
}

}  // extern "C"
