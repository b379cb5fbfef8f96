// Persistent denoise kernel (see persistent.h for the execution model).
//
// Roles inside a CTA (256 threads):
//   warp 0, lane 0  weight producer: bulk copies of every GEMM unit's 16 KB weight chunks, in the
//                   CTA's unit order, into the ring; waits only for free ring slots
//   warp 1, lane 0  MMA issuer: tcgen05.mma (M = 128 features, N = Nt tokens, bf16) per chunk
//                   once its weights and its activation chunk have landed; TMEM accumulator
//   warps 4-7       workers: wait for a unit's inputs (global counters), issue its activation
//                   copies, run the epilogue (split-K exchange, RoPE / residual / GeLU), the
//                   attention units and the per-token final + in-proj units
// Every wait is bounded; a wait that gives up latches the status word, raises the abort counter
// (every CTA leaves its loops), and the CTA drains its copies in flight before it returns.
#include <algorithm>
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "persistent.h"
#include "sm100.h"
#include "tc_device.h"
#include "tc_kernels.h"

namespace fr {
namespace pk {
namespace {

using namespace fr::sm100;
using namespace fr::tc;

constexpr uint32_t CHUNK = BM * KCB;     // one weight chunk: 128 rows x 128 B
constexpr int WK0 = 4;                   // first worker warp
constexpr int ATT_LD_PAD = 8;

// Optional per-unit timestamps (globaltimer), compiled in only with -DFR_PK_TIMELINE for
// performance analysis: per CTA, a 12-word record per worker unit (tag, then the times of its
// steps, the last word its end) and a 4-word record per GEMM unit of the MMA warp; the product
// build has none of this code.
#ifdef FR_PK_TIMELINE
constexpr int PKT_W = 12;                // words per record: tag, then up to 11 timestamps
__device__ unsigned long long* g_pk_tl = nullptr;
__device__ unsigned g_pk_tl_words = 0;   // words per CTA (worker records, then MMA records from the middle)
#define PKT_DECL unsigned long long pkt_[PKT_W] = {0};
#define PKT(i) do { if (c.wt == 0) pkt_[i] = globaltimer(); } while (0)
#define PKT_TAG(v) do { pkt_[0] = (v); } while (0)
#define PKT_FLUSH() do { if (c.wt == 0 && g_pk_tl) { pkt_[PKT_W - 1] = globaltimer(); \
    const unsigned o_ = c.tl_n * PKT_W; if (o_ + PKT_W <= g_pk_tl_words / 2) \
      for (int q_ = 0; q_ < PKT_W; ++q_) g_pk_tl[static_cast<size_t>(c.cta) * g_pk_tl_words + o_ + q_] = pkt_[q_]; \
    ++c.tl_n; } } while (0)
#define PKX_DECL unsigned long long pkx_[PKT_W] = {0};
#define PKX(i) do { if (c.wt == 0) pkx_[i] = globaltimer(); } while (0)
#define PKX_FLUSH(tagv) do { if (c.wt == 0 && g_pk_tl) { pkx_[0] = (tagv); \
    const unsigned o_ = c.tl_n * PKT_W; if (o_ + PKT_W <= g_pk_tl_words / 2) \
      for (int q_ = 0; q_ < PKT_W; ++q_) g_pk_tl[static_cast<size_t>(c.cta) * g_pk_tl_words + o_ + q_] = pkx_[q_]; \
    ++c.tl_n; } } while (0)
// MMA warp: per GEMM unit, (tag, first weight chunk ready, first activation chunk ready, last MMA issued)
#define PKM_REC(tag, t1, t2, t3) do { if (g_pk_tl) { const unsigned o_ = g_pk_tl_words / 2 + mrec * 4; \
    if (o_ + 4 <= g_pk_tl_words) { unsigned long long* r_ = g_pk_tl + static_cast<size_t>(cta) * g_pk_tl_words + o_; \
      r_[0] = (tag); r_[1] = (t1); r_[2] = (t2); r_[3] = (t3); } ++mrec; } } while (0)
#else
#define PKT_DECL
#define PKT(i) do {} while (0)
#define PKT_TAG(v) do {} while (0)
#define PKT_FLUSH() do {} while (0)
#define PKM_REC(tag, t1, t2, t3) do {} while (0)
#define PKX_DECL
#define PKX(i) do {} while (0)
#define PKX_FLUSH(tagv) do {} while (0)
#endif

static_assert(sizeof(PkArgs) % 4 == 0, "argument block copied by words");

struct PkSmem {
  uint64_t wfull[PK_MAX_RING], wempty[PK_MAX_RING];
  uint64_t bfull;                   // the unit's activation chunks landed (one copy per unit)
  uint64_t accfull, accempty, fin, stage;
  uint32_t tmem_base;
  int abort;
  float rstd[PK_MAX_T];
  float w_sh[PK_MAX_C][PK_MAX_T];   // attention merge weights of the owned rows
  float inv_den[PK_MAX_T];
  float part[4][32];                // per-warp sums of squares of 128-feature blocks (D <= 4096)
  float xrow[64];                   // x of the token of a final / in-proj unit (A <= 64)
  int staged;                       // worker 0 issued copies on the stage barrier: wait for them
};

__device__ __forceinline__ void wk_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ bool reached(uint32_t v, uint32_t target) { return static_cast<int>(v - target) >= 0; }

// Bounded mbarrier wait that also gives up when the CTA aborts.
__device__ __forceinline__ bool pk_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t spin = 0;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 31) == 31) {
      if (*abort) return false;
      if (globaltimer() - t0 > WAIT_LIMIT_NS) return false;
    }
  }
}

// Bounded wait on a global counter written by other CTAs (acquire on success).
__device__ __forceinline__ bool wait_counter(const unsigned* p, uint32_t target, unsigned long long limit,
                                             const unsigned* abort_g, volatile int* abort_s) {
  if (reached(ld_acquire_gpu(p), target)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t spin = 0;; ++spin) {
    if (reached(ld_acquire_gpu(p), target)) return true;
    if ((spin & 15) == 15) {
      if (*abort_s || ld_relaxed_gpu(abort_g) != 0) return false;
    }
    if (globaltimer() - t0 > limit) return false;
  }
}

__device__ __forceinline__ int first_unit(int cta, int base, int G) {
  const int u = cta - base;
  return u < 0 ? u + G : u;
}

__device__ __forceinline__ float bf16r(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Number of unit completions that precede a phase instance: stage 0..4 = QKV, ATT, O, GU, DN of
// (step k, layer l); stage 5 = the final/in-proj phase after step k.
__device__ __forceinline__ uint32_t before(const PkArgs& a, int k, int l, int stage) {
  const uint32_t Uq = a.g[PG_QKV].units, Ua = a.att_units, Uo = a.g[PG_O].units, Ug = a.g[PG_GU].units,
                 Ud = a.g[PG_DN].units;
  const uint32_t per_layer = Uq + Ua + Uo + Ug + Ud;
  const uint32_t per_step = a.L * per_layer + a.T;
  uint32_t pre = 0;
  if (stage >= 1) pre += Uq;
  if (stage >= 2) pre += Ua;
  if (stage >= 3) pre += Uo;
  if (stage >= 4) pre += Ug;
  const uint32_t base = a.T + static_cast<uint32_t>(k) * per_step;
  return stage == 5 ? base + a.L * per_layer : base + static_cast<uint32_t>(l) * per_layer + pre;
}

struct Ctx {
  const PkArgs& a;
  PkSmem& sh;
  uint8_t* dsm;
  int cta, wt, ww, lane;
  uint32_t nb;      // activation copies issued (one per GEMM unit)
  uint32_t acc;     // accumulators consumed
  uint32_t stage;   // uses of the stage barrier
  uint32_t tl_n;    // timeline records written (instrumented builds)
};

__device__ void fail(Ctx& c, uint32_t where) {
  if (!c.sh.abort) report_timeout(c.a.status, where | (static_cast<uint32_t>(c.cta) << 16));
  atomicExch(c.a.ctr + CTR_ABORT, 1u);
  c.sh.abort = 1;
}

// Worker thread 0 waits for `target` completions; every worker returns whether to go on.
__device__ bool dep_wait(Ctx& c, uint32_t target, uint32_t where) {
  if (c.wt == 0) {
    if (!wait_counter(c.a.ctr + CTR_DONE, target, c.a.flag_limit_ns, c.a.ctr + CTR_ABORT, &c.sh.abort))
      fail(c, where);
    fence_proxy_async_global();
  }
  wk_sync();
  return !c.sh.abort;
}

// End of a unit: its outputs are visible to other CTAs' bulk copies, then it counts as done.
__device__ void unit_done(Ctx& c) {
  fence_proxy_async_global();
  fence_proxy_async_smem();   // the next job's bulk copies overwrite what this one used in shared memory
  wk_sync();
  if (c.wt == 0) red_release_gpu_add(c.a.ctr + CTR_DONE, 1u);
}

// ---------------------------------------------------------------------------------------------- GEMM units

__device__ __noinline__ bool gemm_unit(Ctx& c, int pg, int k, int l, int u) {
  const PkArgs& a = c.a;
  const PkGemm& gp = a.g[pg];
  const int stage = pg == PG_QKV ? 0 : pg + 1;
  PKT_DECL
  PKT_TAG(static_cast<unsigned long long>(pg) | (static_cast<unsigned long long>(k) << 8) |
          (static_cast<unsigned long long>(l) << 16) | (static_cast<unsigned long long>(u) << 32));
  PKT(1);
  const int it = k * a.L + l;
  const int S = gp.S, mb = u / S, ks = u % S;
  const int kc0 = ks * gp.NKC / S, kc1 = (ks + 1) * gp.NKC / S, nk = kc1 - kc0;
  const int Nt = a.Nt, T = a.T;
  const uint32_t btile = static_cast<uint32_t>(Nt) * KCB;
  uint8_t* ureg = c.dsm + a.u_off;
  float2* rope_sh = reinterpret_cast<float2*>(c.dsm + a.rope_off);
  const int half = a.dh >> 1;
  // QKV: the m-block's (cos, sin) pairs at every action position (static: before the wait)
  if (pg == PG_QKV && mb < a.MB_rot) {
    for (int idx = c.wt; idx < a.H * 64; idx += PK_WORKERS) {
      const int i = idx >> 6, p = idx & 63;
      const int j = (mb * 64 + p) % half, pos = a.P + i;
      rope_sh[idx] = make_float2(a.rope_cos[pos * half + j], a.rope_sin[pos * half + j]);
    }
  }
  // inputs of the phase ready: the unit's activation chunks, one copy into the B region
  if (c.wt == 0) {
    bool ok = wait_counter(a.ctr + CTR_DONE, before(a, k, l, stage), a.flag_limit_ns, a.ctr + CTR_ABORT, &c.sh.abort);
    if (!ok) fail(c, 0x1100 + pg);
    PKT(2);
    if (ok) {
      // the unit's chunks are contiguous in global memory and in the B region: one copy.  The region
      // is free: the previous unit's MMAs completed before its epilogue reused it.
      fence_proxy_async_global();
      mbar_arrive_expect_tx(&c.sh.bfull, nk * btile);
      bulk_g2s(ureg, gp.act + static_cast<size_t>(kc0) * btile, nk * btile, &c.sh.bfull);
      ++c.nb;
    }
    PKT(3);
  }
  wk_sync();
  if (c.sh.abort) return false;
  // deferred RMSNorm factor of the tokens (QKV and gate|up read bf16(h * gamma))
  const bool rscale = pg == PG_QKV || pg == PG_GU;
  if (rscale) {
    const float* ssq = pg == PG_QKV ? a.ssq_a : a.ssq_b;
    for (int r = c.wt; r < Nt; r += PK_WORKERS) {
      float rs = 0.f;
      if (r < T) {
        float ss = 0.f;
        for (int q = 0; q < a.MBd; ++q) ss += ssq[static_cast<size_t>(r) * a.ssq_ld + q];
        rs = 1.0f / sqrtf(ss / a.D + a.eps);
      }
      c.sh.rstd[r] = rs;
    }
  }
  PKT(4);
  // accumulator of this unit
  if (!pk_wait(&c.sh.accfull, c.acc & 1, &c.sh.abort)) {
    if (c.wt == 0) fail(c, 0x1120 + pg);
    return false;
  }
  tc_fence_after();
  PKT(5);
  const uint32_t tacc = c.sh.tmem_base;
  float* red = reinterpret_cast<float*>(ureg);   // S == 1: [Nt][RED_LD]; S > 1: [T][BM] (the partial tile)
  {
    const int row = c.ww * 32 + c.lane;
    for (int c0 = 0; c0 < Nt; c0 += 64) {
      uint32_t v[4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c0 + 16 * q < Nt) tmem_ld16_nowait(tacc + (static_cast<uint32_t>(c.ww * 32) << 16) + c0 + 16 * q, v[q]);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c0 + 16 * q < Nt)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = c0 + 16 * q + j;
            if (S == 1) red[tok * RED_LD + row] = __uint_as_float(v[q][j]);
            else if (tok < T) red[tok * BM + row] = __uint_as_float(v[q][j]);
          }
    }
  }
  tc_fence_before();
  mbar_arrive(&c.sh.accempty);   // 128 arrivals: the MMA warp may start the next unit
  ++c.acc;
  const int tok0 = ks * Nt / S, tok1 = (ks + 1) * Nt / S;
  const int TS = (Nt + S - 1) / S;
  float* xst = reinterpret_cast<float*>(ureg);                        // S > 1: [S][TS][BM]
  float* hst = reinterpret_cast<float*>(c.dsm + a.hrow_off);          // S > 1 residual: [2][TS][64]
  const bool resid = pg == PG_O || pg == PG_DN;
  if (S > 1) {
    // partial tile -> scratch; once the m-block's S partials are in, this unit's token slice of each
    float* xs = a.xscratch + static_cast<size_t>(mb) * S * Nt * BM;
    fence_proxy_async_smem();
    wk_sync();
    PKT(6);
    if (c.wt == 0) {
      c.sh.staged = 0;
      bulk_s2g(xs + static_cast<size_t>(ks) * Nt * BM, red, static_cast<uint32_t>(T) * BM * 4u);
      bulk_commit();
      bulk_wait_all();
      fence_proxy_async_global();
      PKT(7);
      unsigned* rc = a.ctr + CTR_RED + pg * PK_MAX_MB + mb;
      red_release_gpu_add(rc, 1u);
      if (!wait_counter(rc, static_cast<uint32_t>(S) * (it + 1), a.flag_limit_ns, a.ctr + CTR_ABORT, &c.sh.abort)) {
        fail(c, 0x1130 + pg);
      } else {
        PKT(8);
        fence_proxy_async_global();
        const uint32_t sb = static_cast<uint32_t>(tok1 - tok0) * BM * 4u;
        const uint32_t hb = resid ? static_cast<uint32_t>(tok1 - tok0) * 256u : 0u;
        mbar_arrive_expect_tx(&c.sh.stage, S * sb + 2 * hb);
        for (int s2 = 0; s2 < S; ++s2)
          bulk_g2s(xst + static_cast<size_t>(s2) * TS * BM, xs + (static_cast<size_t>(s2) * Nt + tok0) * BM, sb,
                   &c.sh.stage);
        if (resid)
          for (int q = 0; q < 2; ++q)
            bulk_g2s(hst + static_cast<size_t>(q) * TS * 64, a.h + ((static_cast<size_t>(2 * mb + q)) * Nt + tok0) * 64,
                     hb, &c.sh.stage);
        c.sh.staged = 1;
      }
    }
    wk_sync();
    if (c.sh.staged) {   // copies in flight into this CTA's shared memory: wait for them even when aborting
      const bool got = mbar_wait(&c.sh.stage, c.stage & 1, WAIT_LIMIT_NS);
      ++c.stage;
      if (!got && c.wt == 0) fail(c, 0x1140 + pg);
    }
    wk_sync();
    if (c.sh.abort) return false;
  } else {
    wk_sync();
  }
  PKT(9);
  // split-K sum of N consecutive rows of token tok in rank order, times the deferred rstd
  auto vals = [&](int tok, int row, float* out, int N) {
    const float sc = rscale ? c.sh.rstd[tok] : 1.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (S == 1) {
      for (int e = 0; e < N; ++e) acc[e] = red[tok * RED_LD + row + e];
    } else {
      for (int s2 = 0; s2 < S; ++s2) {
        const float* p = xst + (static_cast<size_t>(s2) * TS + (tok - tok0)) * BM + row;
        for (int e = 0; e < N; ++e) acc[e] += p[e];
      }
    }
    for (int e = 0; e < N; ++e) out[e] = acc[e] * sc;
  };
  const float* gains = a.gains + static_cast<size_t>(l) * 2 * a.D;   // [g1 | g2] of layer l
  if (pg == PG_QKV) {
    __nv_bfloat16* kvk = a.kv_k + static_cast<size_t>(l) * a.kv_layer_elems;
    __nv_bfloat16* kvv = a.kv_v + static_cast<size_t>(l) * a.kv_layer_elems;
    if (mb < a.MB_rot) {
      const int p = c.lane * 2;
      const int pi = mb * 64 + p, head = pi / half, j = pi % half;
      for (int tok = tok0 + c.ww; tok < tok1 && tok < T; tok += 4) {
        const int b = tok / a.H, i = tok % a.H, pos = a.P + i;
        const float4 r4 = *reinterpret_cast<const float4*>(rope_sh + i * 64 + p);
        float lo[2], hi[2];
        vals(tok, p, lo, 2);
        vals(tok, p + 64, hi, 2);
        const float r00 = lo[0] * r4.x - hi[0] * r4.y, r10 = lo[0] * r4.y + hi[0] * r4.x;
        const float r01 = lo[1] * r4.z - hi[1] * r4.w, r11 = lo[1] * r4.w + hi[1] * r4.z;
        const bool isq = head < a.Hq;
        const size_t o = isq ? ((static_cast<size_t>(b) * a.Hq + head) * a.H + i) * a.dh
                             : ((static_cast<size_t>(b) * a.Hkv + (head - a.Hq)) * a.S_max + pos) * a.dh;
        __nv_bfloat16* dst = (isq ? a.q : kvk) + o;
        if (in_bounds(a.status, o + j + half + 1, isq ? a.ext.q : a.ext.kv, isq ? 0xA005 : 0xA006)) {
          *reinterpret_cast<uint32_t*>(dst + j) = pack_bf16x2(r00, r01);
          *reinterpret_cast<uint32_t*>(dst + j + half) = pack_bf16x2(r10, r11);
        }
      }
    } else {
      const int row = c.lane * 4;
      const int idx = (mb - a.MB_rot) * BM + row;
      const int g = idx / a.dh, d = idx % a.dh;
      for (int tok = tok0 + c.ww; tok < tok1 && tok < T; tok += 4) {
        const int b = tok / a.H, i = tok % a.H, pos = a.P + i;
        float v4[4];
        vals(tok, row, v4, 4);
        const size_t vo = ((static_cast<size_t>(b) * a.Hkv + g) * a.S_max + pos) * a.dh + d;
        if (in_bounds(a.status, vo + 3, a.ext.kv, 0xA007))
          *reinterpret_cast<uint2*>(kvv + vo) = make_uint2(pack_bf16x2(v4[0], v4[1]), pack_bf16x2(v4[2], v4[3]));
      }
    }
  } else if (pg == PG_GU) {
    const int p = c.lane * 2;
    const int f = mb * 64 + p;
    if (f < a.F)
      for (int tok = tok0 + c.ww; tok < tok1 && tok < T; tok += 4) {
        float g[2], up[2];
        vals(tok, p, g, 2);
        vals(tok, p + 64, up, 2);
        const size_t uo = btile_offset(tok, 2 * f, Nt, a.NKC_u);
        if (in_bounds(a.status, uo + 3, a.ext.ubuf, 0xA004))
          *reinterpret_cast<uint32_t*>(a.ubuf + uo) = pack_bf16x2(gelu_tanh(g[0]) * up[0], gelu_tanh(g[1]) * up[1]);
      }
  } else {   // residual: h += update; sum of squares for the next norm; bf16(h * gamma_next)
    const int row = c.lane * 4;
    const int f = mb * BM + row;
    const bool fok = f < a.D;
    float* ssq_out = pg == PG_O ? a.ssq_b : a.ssq_a;
    const float* g_next = pg == PG_O ? gains + a.D
                        : (l + 1 < a.L ? a.gains + static_cast<size_t>(l + 1) * 2 * a.D : nullptr);
    float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (g_next && fok) g4 = *reinterpret_cast<const float4*>(g_next + f);
    for (int tok = tok0 + c.ww; tok < tok1 && tok < T; tok += 4) {
      float sq = 0.f;
      if (fok) {
        float4 hv = S > 1 ? *reinterpret_cast<const float4*>(hst + ((row >> 6) * TS + (tok - tok0)) * 64 + (row & 63))
                          : *reinterpret_cast<const float4*>(a.h + htile_offset(tok, f, Nt, a.KB));
        float d4[4];
        vals(tok, row, d4, 4);
        hv.x += d4[0];
        hv.y += d4[1];
        hv.z += d4[2];
        hv.w += d4[3];
        sq = ((hv.x * hv.x + hv.y * hv.y) + hv.z * hv.z) + hv.w * hv.w;
        const size_t ho = htile_offset(tok, f, Nt, a.KB);
        if (in_bounds(a.status, ho + 3, a.ext.h, 0xA001)) *reinterpret_cast<float4*>(a.h + ho) = hv;
        const size_t xo = btile_offset(tok, 2 * f, Nt, a.NKC_x);
        if (g_next && in_bounds(a.status, xo + 7, a.ext.xbuf, 0xA002))
          *reinterpret_cast<uint2*>(a.xbuf + xo) =
              make_uint2(pack_bf16x2(hv.x * g4.x, hv.y * g4.y), pack_bf16x2(hv.z * g4.z, hv.w * g4.w));
      }
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      const size_t so = static_cast<size_t>(tok) * a.ssq_ld + mb;
      if (c.lane == 0 && in_bounds(a.status, so, a.ext.ssq, 0xA003)) ssq_out[so] = sq;
    }
  }
  PKT(10);
  unit_done(c);
  PKT_FLUSH();
  return true;
}

// ---------------------------------------------------------------------------------------------- attention units

// One (sample b, query head j, key chunk ch) unit: warp-level bf16 MMA over the chunk's keys with
// an online softmax (the flash-decoding split), the chunk's (O, max, sum) rows to the scratch, and
// the merge of the rows this chunk owns over all chunks of the head in chunk order.
template <int DH>
__device__ __noinline__ bool attn_unit(Ctx& c, int k, int l, int u) {
  const PkArgs& a = c.a;
  constexpr int LD = DH + ATT_LD_PAD;
  constexpr int OLD = DH + 4;
  constexpr int VPR = DH / 8;
  const int C = a.C, ch = u % C, j = (u / C) % a.Hq, b = u / (C * a.Hq);
  const int it = k * a.L + l;
  const int g = (j * a.Hkv) / a.Hq;
  const int H = a.H, Hp = (H + 15) & ~15;
  const int S_keys = a.P + H;
  const int key0 = ch * a.KC;
  const int nkeys = min(a.KC, S_keys - key0);
  uint8_t* ureg = c.dsm + a.u_off;
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(ureg);
  __nv_bfloat16* Ks = Qs + Hp * LD;
  __nv_bfloat16* Vs = Ks + a.KC * LD;
  float* Obuf = reinterpret_cast<float*>(ureg);
  const size_t kvo = static_cast<size_t>(l) * a.kv_layer_elems + (static_cast<size_t>(b) * a.Hkv + g) * a.S_max * DH;
  const __nv_bfloat16* kg = a.kv_k + kvo;
  const __nv_bfloat16* vg = a.kv_v + kvo;
  float* xs = a.xscratch + (static_cast<size_t>(b) * a.Hq + j) * C * H * OLD;
  const int tid = c.wt, warp = c.ww, lane = c.lane;
  PKT_DECL
  PKT_TAG(4ull | (static_cast<unsigned long long>(k) << 8) | (static_cast<unsigned long long>(l) << 16) |
          (static_cast<unsigned long long>(u) << 32));
  PKT(1);
  // cached keys/values do not depend on this step: start their loads before the wait
  for (int itv = tid; itv < a.KC * VPR; itv += PK_WORKERS) {
    const int r = itv / VPR, v = itv % VPR;
    const int key = key0 + r;
    if (key < a.P || r >= nkeys) {
      const bool ok = r < nkeys;
      cp_async16(Ks + r * LD + v * 8, kg + static_cast<size_t>(ok ? key : 0) * DH + v * 8, ok);
      cp_async16(Vs + r * LD + v * 8, vg + static_cast<size_t>(ok ? key : 0) * DH + v * 8, ok);
    }
  }
  cp_async_commit();
  if (!dep_wait(c, before(a, k, l, 1), 0x1200)) {
    cp_async_wait_all();
    return false;
  }
  PKT(2);
  for (int itv = tid; itv < a.KC * VPR; itv += PK_WORKERS) {
    const int r = itv / VPR, v = itv % VPR;
    const int key = key0 + r;
    if (key >= a.P && r < nkeys) {
      cp_async16(Ks + r * LD + v * 8, kg + static_cast<size_t>(key) * DH + v * 8, true);
      cp_async16(Vs + r * LD + v * 8, vg + static_cast<size_t>(key) * DH + v * 8, true);
    }
  }
  const __nv_bfloat16* qg = a.q + ((static_cast<size_t>(b) * a.Hq + j) * H) * DH;
  for (int itv = tid; itv < Hp * VPR; itv += PK_WORKERS) {
    const int r = itv / VPR, v = itv % VPR;
    cp_async16(Qs + r * LD + v * 8, qg + static_cast<size_t>(r < H ? r : 0) * DH + v * 8, r < H);
  }
  cp_async_commit();
  cp_async_wait_all();
  wk_sync();

  const int gq = lane >> 2, tq = lane & 3;
  const float sl2 = a.scale * 1.4426950408889634f;
  const int rg = warp;
  const bool active = rg < Hp / 16;
  float oacc[DH / 8][4];
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  if (active) {
#pragma unroll
    for (int n = 0; n < DH / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
    const uint32_t qa = smem_u32(Qs + (rg * 16 + (lane & 15)) * LD + (lane >> 4) * 8);
    for (int kb = 0; kb < nkeys; kb += ATTN_SUBK) {
      float sacc[ATTN_SUBK / 8][4];
#pragma unroll
      for (int n = 0; n < ATTN_SUBK / 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(qa + kk * 32, a0, a1, a2, a3);
#pragma unroll
        for (int n = 0; n < ATTN_SUBK / 8; ++n) {
          uint32_t b0, b1;
          const uint32_t ka = smem_u32(Ks + (kb + n * 8 + (lane & 7)) * LD + kk * 16 + ((lane >> 3) & 1) * 8);
          ldsm_x2(ka, b0, b1);
          mma16816(sacc[n], a0, a1, a2, a3, b0, b1);
        }
      }
      float mnew[2] = {mrow[0], mrow[1]};
#pragma unroll
      for (int n = 0; n < ATTN_SUBK / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = kb + n * 8 + tq * 2 + (e & 1);
          float v = sacc[n][e] * sl2;
          if (key >= nkeys) v = -INFINITY;
          sacc[n][e] = v;
          mnew[e >> 1] = fmaxf(mnew[e >> 1], v);
        }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mnew[h2] = fmaxf(mnew[h2], __shfl_xor_sync(0xffffffffu, mnew[h2], 1));
        mnew[h2] = fmaxf(mnew[h2], __shfl_xor_sync(0xffffffffu, mnew[h2], 2));
      }
      float corr[2], psum[2] = {0.f, 0.f};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) corr[h2] = exp2f(mrow[h2] - mnew[h2]);
#pragma unroll
      for (int n = 0; n < ATTN_SUBK / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = exp2f(sacc[n][e] - mnew[e >> 1]);
          sacc[n][e] = p;
          psum[e >> 1] += p;
        }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        psum[h2] += __shfl_xor_sync(0xffffffffu, psum[h2], 1);
        psum[h2] += __shfl_xor_sync(0xffffffffu, psum[h2], 2);
        lrow[h2] = lrow[h2] * corr[h2] + psum[h2];
        mrow[h2] = mnew[h2];
      }
#pragma unroll
      for (int n = 0; n < DH / 8; ++n) {
        oacc[n][0] *= corr[0];
        oacc[n][1] *= corr[0];
        oacc[n][2] *= corr[1];
        oacc[n][3] *= corr[1];
      }
#pragma unroll
      for (int kk = 0; kk < ATTN_SUBK / 16; ++kk) {
        const uint32_t p0 = pack_bf16x2(sacc[2 * kk][0], sacc[2 * kk][1]);
        const uint32_t p1 = pack_bf16x2(sacc[2 * kk][2], sacc[2 * kk][3]);
        const uint32_t p2 = pack_bf16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
        const uint32_t p3 = pack_bf16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
        const uint32_t va0 = smem_u32(Vs + (kb + kk * 16 + (lane & 15)) * LD);
#pragma unroll
        for (int n = 0; n < DH / 8; ++n) {
          uint32_t b0, b1;
          ldsm_x2_t(va0 + n * 16, b0, b1);
          mma16816(oacc[n], p0, p1, p2, p3, b0, b1);
        }
      }
    }
  }
  wk_sync();   // every warp is done with Q/K/V: the partial rows overwrite them
  PKT(3);
  if (active) {
    const int r0 = rg * 16 + gq;
#pragma unroll
    for (int n = 0; n < DH / 8; ++n) {
      const int col = n * 8 + tq * 2;
      *reinterpret_cast<float2*>(Obuf + r0 * OLD + col) = make_float2(oacc[n][0], oacc[n][1]);
      *reinterpret_cast<float2*>(Obuf + (r0 + 8) * OLD + col) = make_float2(oacc[n][2], oacc[n][3]);
    }
    if (tq == 0) {
      *reinterpret_cast<float2*>(Obuf + r0 * OLD + DH) = make_float2(mrow[0], lrow[0]);
      *reinterpret_cast<float2*>(Obuf + (r0 + 8) * OLD + DH) = make_float2(mrow[1], lrow[1]);
    }
  }
  const int r_lo = ch * H / C, r_hi = (ch + 1) * H / C, nr = r_hi - r_lo;
  const int R = (H + C - 1) / C;
  float* stage = reinterpret_cast<float*>(ureg);   // C > 1: [C][R][OLD], this chunk's owned rows of every chunk
  if (C > 1) {
    fence_proxy_async_smem();
    wk_sync();
    if (tid == 0) {
      c.sh.staged = 0;
      bulk_s2g(xs + static_cast<size_t>(ch) * H * OLD, Obuf, static_cast<uint32_t>(H) * OLD * 4u);
      bulk_commit();
      bulk_wait_all();
      fence_proxy_async_global();
      unsigned* ac = a.ctr + CTR_ATT + b * a.Hq + j;
      red_release_gpu_add(ac, 1u);
      if (!wait_counter(ac, static_cast<uint32_t>(C) * (it + 1), a.flag_limit_ns, a.ctr + CTR_ABORT, &c.sh.abort)) {
        fail(c, 0x1210);
      } else if (nr > 0) {
        fence_proxy_async_global();
        const uint32_t sb = static_cast<uint32_t>(nr) * OLD * 4u;
        mbar_arrive_expect_tx(&c.sh.stage, C * sb);
        for (int s2 = 0; s2 < C; ++s2)
          bulk_g2s(stage + static_cast<size_t>(s2) * R * OLD, xs + (static_cast<size_t>(s2) * H + r_lo) * OLD, sb,
                   &c.sh.stage);
        c.sh.staged = 1;
      }
    }
    wk_sync();
    if (c.sh.staged) {   // copies in flight into this CTA's shared memory: wait for them even when aborting
      const bool got = mbar_wait(&c.sh.stage, c.stage & 1, WAIT_LIMIT_NS);
      ++c.stage;
      if (!got && tid == 0) fail(c, 0x1220);
    }
    wk_sync();
    if (c.sh.abort) return false;
  } else {
    wk_sync();
  }
  PKT(4);
  // merge the owned rows over the chunks, in chunk order
  const float* src = C > 1 ? stage : Obuf;
  const size_t sstride = C > 1 ? static_cast<size_t>(R) : 0;
  const int roff = C > 1 ? 0 : r_lo;
  if (tid < nr) {
    float mv[PK_MAX_C], lv[PK_MAX_C];
#pragma unroll
    for (int s = 0; s < PK_MAX_C; ++s) {
      if (s < C) {
        const float2 ml = *reinterpret_cast<const float2*>(src + (s * sstride + roff + tid) * OLD + DH);
        mv[s] = ml.x;
        lv[s] = ml.y;
      } else {
        mv[s] = -INFINITY;
        lv[s] = 0.f;
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < PK_MAX_C; ++s) M = fmaxf(M, mv[s]);
    float den = 0.f;
#pragma unroll
    for (int s = 0; s < PK_MAX_C; ++s)
      if (s < C) {
        const float e = exp2f(mv[s] - M);
        c.sh.w_sh[s][tid] = e;
        den += e * lv[s];
      }
    c.sh.inv_den[tid] = 1.0f / den;
  }
  wk_sync();
  for (int itv = tid; itv < nr * (DH / 8); itv += PK_WORKERS) {
    const int rr = itv / (DH / 8), d0 = (itv % (DH / 8)) * 8;
    float acc8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc8[e] = 0.f;
    for (int s = 0; s < C; ++s) {
      const float w = c.sh.w_sh[s][rr];
      const float* p = src + (s * sstride + roff + rr) * OLD + d0;
      const float4 v0 = *reinterpret_cast<const float4*>(p), v1 = *reinterpret_cast<const float4*>(p + 4);
      acc8[0] += w * v0.x;
      acc8[1] += w * v0.y;
      acc8[2] += w * v0.z;
      acc8[3] += w * v0.w;
      acc8[4] += w * v1.x;
      acc8[5] += w * v1.y;
      acc8[6] += w * v1.z;
      acc8[7] += w * v1.w;
    }
    const float id = c.sh.inv_den[rr];
    const int t = b * H + r_lo + rr;
    const int kidx = j * DH + d0;
    const size_t ob = btile_offset(t, 2 * kidx, a.Nt, a.NKC_o);
    if (in_bounds(a.status, ob + 15, a.ext.obuf, 0xA010))
      *reinterpret_cast<uint4*>(a.obuf + ob) =
          make_uint4(pack_bf16x2(acc8[0] * id, acc8[1] * id), pack_bf16x2(acc8[2] * id, acc8[3] * id),
                     pack_bf16x2(acc8[4] * id, acc8[5] * id), pack_bf16x2(acc8[6] * id, acc8[7] * id));
  }
  PKT(10);
  unit_done(c);
  PKT_FLUSH();
  return true;
}

// ---------------------------------------------------------------------------------------------- final + in-proj units

// Token t: the final norm, out-proj and Euler update of step kf (kf >= 0), then the in-proj and
// time embedding of step kf + 1 (kf + 1 < K): h, its sums of squares, bf16(h * gamma1 of layer 0).
__device__ __noinline__ bool fi_unit(Ctx& c, int kf, int t) {
  const PkArgs& a = c.a;
  const int D = a.D, A = a.A;
  float* hn = reinterpret_cast<float*>(c.dsm + a.u_off);
  PKT_DECL
  PKT_TAG(5ull | (static_cast<unsigned long long>(kf + 1) << 8) | (static_cast<unsigned long long>(t) << 32));
  PKT(1);
  if (kf >= 0) {
    if (!dep_wait(c, before(a, kf, 0, 5), 0x1300)) return false;
    PKT(2);
    float ss = 0.f;
    for (int p = 0; p < a.MBd; ++p) ss += a.ssq_a[static_cast<size_t>(t) * a.ssq_ld + p];
    const float r = 1.0f / sqrtf(ss / D + a.eps);
    for (int d = c.wt; d < D; d += PK_WORKERS) hn[d] = bf16r(a.h[htile_offset(t, d, a.Nt, a.KB)] * r * a.g_f[d]);
    wk_sync();
    const float* x_in = kf == 0 ? a.x0 : a.xs;
    float* x_nx = kf == a.K - 1 ? a.x_out : a.xs;
    for (int i = c.ww; i < A; i += 4) {
      const __nv_bfloat16* wr = a.w_out + static_cast<size_t>(i) * D;
      float acc = 0.f;
      for (int d = c.lane; d < D; d += 32) acc = fmaf(__bfloat162float(wr[d]), hn[d], acc);
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (c.lane == 0) {
        const size_t xi = static_cast<size_t>(t) * A + i;
        const float xn = x_in[xi] + a.dt * (acc + a.b_out[i]);
        if (in_bounds(a.status, xi, a.ext.x, 0xA020)) x_nx[xi] = xn;
        c.sh.xrow[i] = xn;
      }
    }
    wk_sync();
  } else {
    for (int i = c.wt; i < A; i += PK_WORKERS) c.sh.xrow[i] = a.x0[static_cast<size_t>(t) * A + i];
    wk_sync();
  }
  if (kf + 1 < a.K) {
    const int kn = kf + 1;
    const float* temb = a.temb + static_cast<size_t>(kn) * D;
    const float* g1 = a.gains;   // layer 0, first norm
    const int nq = (D + BM - 1) / BM;
    for (int qb = 0; qb < nq; ++qb) {
      const int n = qb * BM + c.wt;
      float hv = 0.f;
      if (n < D) {
        float acc = 0.f;
        for (int i = 0; i < A; ++i) acc = fmaf(__bfloat162float(a.w_in_t[static_cast<size_t>(i) * D + n]), bf16r(c.sh.xrow[i]), acc);
        hv = acc + a.b_in[n] + temb[n];
        const size_t ho = htile_offset(t, n, a.Nt, a.KB), xo = btile_offset(t, 2 * n, a.Nt, a.NKC_x);
        if (in_bounds(a.status, ho, a.ext.h, 0xA021)) a.h[ho] = hv;
        if (in_bounds(a.status, xo + 1, a.ext.xbuf, 0xA022))
          *reinterpret_cast<__nv_bfloat16*>(a.xbuf + xo) = __float2bfloat16_rn(hv * g1[n]);
      }
      float sq = hv * hv;
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (c.lane == 0) c.sh.part[c.ww][qb] = sq;
    }
    wk_sync();
    if (c.wt < nq && in_bounds(a.status, static_cast<size_t>(t) * a.ssq_ld + c.wt, a.ext.ssq, 0xA023))
      a.ssq_a[static_cast<size_t>(t) * a.ssq_ld + c.wt] =
          ((c.sh.part[0][c.wt] + c.sh.part[1][c.wt]) + c.sh.part[2][c.wt]) + c.sh.part[3][c.wt];
  }
  unit_done(c);
  PKT_FLUSH();
  return true;
}

// ---------------------------------------------------------------------------------------------- the kernel

template <int DH>
__global__ void __launch_bounds__(PK_THREADS, 1) k_loop_persistent(const __grid_constant__ PkArgs args) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ PkSmem sh;
  // The unit functions are not inlined and reach the arguments through a reference: a copy in shared
  // memory keeps those reads on-chip (a generic pointer into the parameter space is not known to be
  // read-only, so every use inside a loop would be a reload).
  __shared__ __align__(16) PkArgs a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < static_cast<int>(sizeof(PkArgs) / 4); i += PK_THREADS)
    reinterpret_cast<uint32_t*>(&a)[i] = reinterpret_cast<const uint32_t*>(&args)[i];
  __syncthreads();
  const int cta = blockIdx.x, G = a.G;
  if (tid == 0) {
    for (int s = 0; s < a.ring; ++s) {
      mbar_init(&sh.wfull[s], 1);
      mbar_init(&sh.wempty[s], 1);
    }
    mbar_init(&sh.bfull, 1);
    mbar_init(&sh.accfull, 1);
    mbar_init(&sh.accempty, PK_WORKERS);
    mbar_init(&sh.fin, 1);
    mbar_init(&sh.stage, 1);
    sh.abort = 0;
    sh.staged = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ---------------- weight producer: every GEMM unit of the CTA, in execution order
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      uint32_t n = 0;
      bool ok = true;
      for (int k = 0; k < a.K && ok; ++k)
        for (int l = 0; l < a.L && ok; ++l) {
          const uint8_t* Wl = a.W + static_cast<size_t>(l) * a.layer_bytes;
          for (int pg = 0; pg < 4 && ok; ++pg) {
            const PkGemm& gp = a.g[pg];
            for (int u = first_unit(cta, gp.base, G); u < gp.units && ok; u += G) {
              const int mb = u / gp.S, ks = u % gp.S;
              const int kc0 = ks * gp.NKC / gp.S, kc1 = (ks + 1) * gp.NKC / gp.S;
              const uint8_t* src = Wl + gp.w_off + (static_cast<size_t>(mb) * gp.NKC + kc0) * CHUNK;
              for (int i = 0; i < kc1 - kc0; ++i) {
                const int s = n % a.ring;
                if (n >= static_cast<uint32_t>(a.ring) && !pk_wait(&sh.wempty[s], ((n / a.ring) - 1) & 1, &sh.abort)) {
                  ok = false;
                  break;
                }
                mbar_arrive_expect_tx(&sh.wfull[s], CHUNK);
                bulk_g2s_hint(dsm + s * CHUNK, src + static_cast<size_t>(i) * CHUNK, CHUNK, &sh.wfull[s], pol);
                ++n;
              }
            }
          }
        }
      if (!ok && !sh.abort) {
        report_timeout(a.status, 0x1000 | (static_cast<uint32_t>(cta) << 16));
        atomicExch(a.ctr + CTR_ABORT, 1u);
        sh.abort = 1;
      }
      // the copies issued into this CTA's shared memory land before it leaves
      for (uint32_t i = n > static_cast<uint32_t>(a.ring) ? n - a.ring : 0; i < n; ++i)
        mbar_wait(&sh.wfull[i % a.ring], (i / a.ring) & 1, WAIT_LIMIT_NS);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(FMT_BF16, BM, a.Nt);
      const uint32_t tacc = sh.tmem_base;
      uint32_t n = 0, nb = 0, acc = 0;
#ifdef FR_PK_TIMELINE
      unsigned mrec = 0;
#endif
      bool ok = true;
      for (int k = 0; k < a.K && ok; ++k)
        for (int l = 0; l < a.L && ok; ++l)
          for (int pg = 0; pg < 4 && ok; ++pg) {
            const PkGemm& gp = a.g[pg];
            for (int u = first_unit(cta, gp.base, G); u < gp.units && ok; u += G) {
              const int ks = u % gp.S;
              const int nk = (ks + 1) * gp.NKC / gp.S - ks * gp.NKC / gp.S;
              if (acc > 0 && !pk_wait(&sh.accempty, (acc - 1) & 1, &sh.abort)) {
                ok = false;
                break;
              }
#ifdef FR_PK_TIMELINE
              unsigned long long tw = 0, tb = 0;
#endif
              for (int i = 0; i < nk; ++i, ++n) {
                const int s = n % a.ring;
                if (!pk_wait(&sh.wfull[s], (n / a.ring) & 1, &sh.abort)) {
                  ok = false;
                  break;
                }
#ifdef FR_PK_TIMELINE
                if (i == 0) tw = globaltimer();
#endif
                if (i == 0 && !pk_wait(&sh.bfull, nb & 1, &sh.abort)) {   // the unit's activation chunks
                  ok = false;
                  break;
                }
#ifdef FR_PK_TIMELINE
                if (i == 0) tb = globaltimer();
#endif
                tc_fence_after();
                const uint32_t a0 = smem_u32(dsm + s * CHUNK);
                const uint32_t b0 = smem_u32(dsm + a.u_off + i * a.Nt * KCB);
#pragma unroll
                for (int kk = 0; kk < KCB / 32; ++kk)
                  mma_bf16(tacc, smem_desc(a0 + kk * 2 * BM * 16, BM * 16, 128),
                           smem_desc(b0 + kk * 2 * a.Nt * 16, a.Nt * 16, 128), idesc, (i | kk) != 0);
                mma_commit(&sh.wempty[s]);
              }
              ++nb;
              if (!ok) break;
              mma_commit(&sh.accfull);
              PKM_REC(static_cast<unsigned long long>(pg) | (static_cast<unsigned long long>(k) << 8) |
                          (static_cast<unsigned long long>(l) << 16) | (static_cast<unsigned long long>(u) << 32),
                      tw, tb, globaltimer());
              ++acc;
            }
          }
      if (!ok && !sh.abort) {
        report_timeout(a.status, 0x1001 | (static_cast<uint32_t>(cta) << 16));
        atomicExch(a.ctr + CTR_ABORT, 1u);
        sh.abort = 1;
      }
      mma_commit(&sh.fin);   // every MMA issued has completed before the accumulator is freed
      mbar_wait(&sh.fin, 0, WAIT_LIMIT_NS);
    }
    __syncwarp();
  } else if (warp >= WK0) {
    // ---------------- workers
    Ctx c{a, sh, dsm, cta, tid - WK0 * 32, warp - WK0, lane, 0u, 0u, 0u, 0u};
    bool ok = true;
    for (int t = first_unit(cta, a.fi_base, G); t < a.T && ok; t += G) ok = fi_unit(c, -1, t);
    for (int k = 0; k < a.K && ok; ++k) {
      for (int l = 0; l < a.L && ok; ++l) {
        for (int u = first_unit(cta, a.g[PG_QKV].base, G); u < a.g[PG_QKV].units && ok; u += G)
          ok = gemm_unit(c, PG_QKV, k, l, u);
        for (int u = first_unit(cta, a.att_base, G); u < a.att_units && ok; u += G) ok = attn_unit<DH>(c, k, l, u);
        for (int pg = PG_O; pg <= PG_DN && ok; ++pg)
          for (int u = first_unit(cta, a.g[pg].base, G); u < a.g[pg].units && ok; u += G) ok = gemm_unit(c, pg, k, l, u);
      }
      for (int t = first_unit(cta, a.fi_base, G); t < a.T && ok; t += G) ok = fi_unit(c, k, t);
    }
    // leave nothing in flight: cp.async groups, bulk stores, the last activation copy
    cp_async_wait_all();
    if (c.wt == 0) {
      bulk_wait_all();
      if (c.nb > 0) mbar_wait(&sh.bfull, (c.nb - 1) & 1, WAIT_LIMIT_NS);
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(sh.tmem_base, 64);
  }
  // the last CTA to leave clears the counters for the next call
  if (tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(a.ctr + CTR_EXIT, 1u);
    if (prev == static_cast<unsigned>(G) - 1u) {
      __threadfence();
      for (int w = 0; w < CTR_WORDS; ++w) a.ctr[w] = 0u;
      __threadfence();
    }
  }
}

const void* kernel_for(int dh) {
  if (dh == 64) return reinterpret_cast<const void*>(k_loop_persistent<64>);
  if (dh == 128) return reinterpret_cast<const void*>(k_loop_persistent<128>);
  if (dh == 256) return reinterpret_cast<const void*>(k_loop_persistent<256>);
  return nullptr;
}

}  // namespace

size_t pk_smem_bytes(const PkArgs& a) {
  const int Hp = (a.H + 15) & ~15;
  const size_t att = static_cast<size_t>(Hp) * (a.dh + ATT_LD_PAD) * 2 + 2ull * a.KC * (a.dh + ATT_LD_PAD) * 2;
  const int R = (a.H + a.C - 1) / a.C;
  const size_t merge = std::max(static_cast<size_t>(Hp) * (a.dh + 4) * 4, static_cast<size_t>(a.C) * R * (a.dh + 4) * 4);
  // GEMM units: the B region / epilogue stage, then the RoPE pairs or the residual rows after it
  const size_t rope_end = a.rope_off + static_cast<size_t>(a.H) * 64 * 8;
  const size_t hrow_end = a.hrow_off + 2ull * a.Nt * 64 * 4;   // [2][TS][64], TS <= Nt
  size_t end = std::max(rope_end, hrow_end);
  end = std::max(end, a.u_off + std::max(att, merge));
  end = std::max(end, a.u_off + static_cast<size_t>(a.D) * 4);
  return (end + 1023) & ~size_t(1023);
}

cudaError_t pk_init() {
  cudaError_t e;
  int dev = 0, optin = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  for (int dh : {64, 128, 256}) {
    const void* f = kernel_for(dh);
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, f)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  optin - static_cast<int>(fa.sharedSizeBytes))) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

int pk_max_dynamic_smem() {
  int dev = 0, optin = 0;
  cudaFuncAttributes fa;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, kernel_for(256)) != cudaSuccess)
    return 0;
  return optin - static_cast<int>(fa.sharedSizeBytes);
}

int pk_max_blocks_per_sm(const PkArgs& a) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel_for(a.dh), PK_THREADS, pk_smem_bytes(a)) != cudaSuccess)
    return 0;
  return n;
}

cudaError_t pk_launch(const PkArgs& a, cudaStream_t s) {
  const void* f = kernel_for(a.dh);
  if (!f) return cudaErrorInvalidValue;
  PkArgs copy = a;
  void* args[] = {&copy};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.G);
  cfg.blockDim = dim3(PK_THREADS);
  cfg.dynamicSmemBytes = pk_smem_bytes(a);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident at once: they wait on one another
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, f, args);
}

}  // namespace pk
}  // namespace fr

#ifdef FR_PK_TIMELINE
// Instrumented builds: point the persistent kernel's timeline at dev_buf (words_per_cta 64-bit words
// per CTA; nullptr switches it off).
extern "C" int fr_debug_pk_timeline(unsigned long long* dev_buf, unsigned words_per_cta) {
  cudaMemcpyToSymbol(fr::pk::g_pk_tl, &dev_buf, sizeof(dev_buf));
  cudaMemcpyToSymbol(fr::pk::g_pk_tl_words, &words_per_cta, sizeof(words_per_cta));
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : -4;
}
#endif
