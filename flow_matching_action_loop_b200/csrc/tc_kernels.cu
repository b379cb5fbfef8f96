// Tensor-core kernels of the action-expert loop (sm_100a).
//
// GEMM (swap-AB): D[128 features x Nt tokens] = W_tile[128 x K] * act[Nt x K]^T on tcgen05
//   with the accumulator in tensor memory.  Both operands arrive by bulk copy (TMA
//   engine): the weight chunks (pre-tiled by the packer, one 16 KB block per chunk) are
//   issued before the kernel waits on its predecessor; the activation chunks after it.
//   For the QKV and gate|up projections the activation is the raw fp32 residual h and
//   warps 2-7 turn it into RMSNorm(h)*gamma (bf16 or e4m3) in shared memory (FlashRT
//   walkthrough, component 8: norm and residual+norm+quant fusion).  Split-K is a
//   thread-block cluster: each CTA pushes the token slices of its partial tile to their
//   owners with bulk shared-to-shared copies, and each owner sums its slices in rank
//   order (deterministic).  Fused epilogues:
//     EPI_QKV   QKV split + rotate-half RoPE, q to its buffer, k/v into the KV cache
//     EPI_RESID residual add into h and the per-token sum of squares of the new h
//     EPI_GELU  GeLU(tanh)(gate) * up, quantised, written as the down projection's operand
//   (PhyAI page, optimisation paragraph: fused QKV and merged gate|up GEMMs.)
//
// Attention: one cluster per (sample, query head), one CTA per key chunk (flash-decoding
//   split over keys).  Warp-level bf16 MMA computes scores and P*V with an online softmax
//   over 64-key sub-chunks; the chunks' (O, max, sum) rows are pushed to their owner CTA by
//   bulk copies and merged with log-sum-exp weights in rank order.
#include <algorithm>
#include <mutex>
#include <type_traits>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"
#include "sm100.h"
#include "tc_kernels.h"
#include "tc_device.h"

namespace fr {
namespace tc {
namespace {

using namespace fr::sm100;

// Optional phase timestamps (globaltimer per CTA), compiled in only with -DFR_TIMELINE for
// performance analysis; the product build has none of this code.
#ifdef FR_TIMELINE
__device__ unsigned long long* g_tl = nullptr;   // [cap][16]: kind, cta, t0..t13
__device__ unsigned g_tl_count = 0;
__device__ unsigned g_tl_cap = 0;
// The record pointer is resolved once per CTA into shared memory, so that a timestamp costs a
// clock read and a store, not a global load ahead of the clock read.
#define TL_DECL __shared__ unsigned long long* tl_rec_;
#define TL_BEGIN(kind)                                                                          \
  do {                                                                                          \
    if (threadIdx.x == 0) {                                                                     \
      const unsigned long long t0_ = fr::sm100::globaltimer();                                 \
      unsigned long long* base_ = g_tl;                                                         \
      const unsigned slot_ = base_ ? atomicAdd(&g_tl_count, 1u) : 0xFFFFFFFFu;                 \
      tl_rec_ = (base_ && slot_ < g_tl_cap) ? base_ + static_cast<size_t>(slot_) * 16 : nullptr; \
      if (tl_rec_) {                                                                            \
        tl_rec_[0] = (kind);                                                                    \
        tl_rec_[1] = blockIdx.x | (blockIdx.y << 10) | (blockIdx.z << 20);                      \
        tl_rec_[2] = t0_;                                                                       \
      }                                                                                         \
    }                                                                                           \
    __syncthreads();                                                                            \
  } while (0)
#define TL(k)                                                                                   \
  do {                                                                                          \
    const unsigned long long t_ = fr::sm100::globaltimer();                                     \
    unsigned long long* r_ = tl_rec_;                                                           \
    if (r_) r_[2 + (k)] = t_;                                                                   \
  } while (0)
#else
#define TL_DECL
#define TL_BEGIN(kind) do {} while (0)
#define TL(k) do {} while (0)
#endif

constexpr int CONV_THREADS = 192;                                  // warps 2-7

__device__ __forceinline__ void conv_sync() { asm volatile("bar.sync 1, 192;" ::: "memory"); }

// ================================================================== GEMM

struct GemmSmem {
  uint64_t full_a[MAX_STAGES];
  uint64_t full_b[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t done;
  uint64_t hbar;      // residual rows of this CTA's tokens (EPI_RESID, S > 1)
  uint64_t xbar;      // split-K slices of this CTA's tokens (S > 1)
  uint64_t raw_a[MAX_STAGES];   // w4: raw 4-bit chunk landed
  uint64_t sbar;      // w4: the scales of this CTA's k-range landed
  uint32_t tmem_base;
  float rstd[NT_MAX];
  float ssq_part[2][4];
};

struct GemmGeom {
  uint32_t a_bytes, breg, slot, ring, gamma_off, recv_off;
  uint32_t rawa_off, scl_off;   // w4: raw 4-bit chunks [stages][4 KB], bf16 scales [groups][128]
  int TS;
};

constexpr uint32_t W4_CHUNK = BM * KCB / 4;   // 4-bit codes of one 128 x 64 weight chunk (4 KB)

// 4-bit scale groups (128 inputs = two 64-element chunks) touched by chunks kc0 .. kc0+nk-1
__host__ __device__ __forceinline__ int w4_groups(int kc0, int nk) { return nk > 0 ? (kc0 + nk - 1) / 2 - kc0 / 2 + 1 : 0; }

__host__ __device__ __forceinline__ GemmGeom gemm_geom(int Nt, int stages, int b_kind, int fp8, int S, int nk,
                                                       int w4 = 0, int kc0 = 0, int kpu = 1) {
  GemmGeom g;
  g.a_bytes = BM * KCB * static_cast<uint32_t>(kpu);   // one ring slot: kpu consecutive k-chunks
  // (B_NORM: the converters read h from global memory straight into the B slot)
  g.breg = static_cast<uint32_t>(Nt) * KCB * static_cast<uint32_t>(kpu);
  g.slot = g.a_bytes + g.breg;
  g.ring = g.slot * static_cast<uint32_t>(stages);
  g.TS = (Nt + S - 1) / S;
  // S > 1: residual rows (2 x TS x 64 floats) live past the ring, the gamma slice and the
  // split-K slices: they land while the ring is still in use and are read after the split-K
  // slices (S x TS x 128 floats, overlaying the ring from offset 0) have landed.
  const uint32_t kel = fp8 ? KCB : KCB / 2;
  g.rawa_off = g.ring;
  g.scl_off = g.rawa_off + (w4 ? static_cast<uint32_t>(stages) * W4_CHUNK : 0u);
  // scale groups of any k-range of nk chunks: at most nk/2 + 1 (one more when kc0 is odd)
  const uint32_t scl_bytes = w4 ? static_cast<uint32_t>(w4_groups(kc0, nk) > nk / 2 + 1 ? w4_groups(kc0, nk) : nk / 2 + 1) * BM * 2u : 0u;
  g.gamma_off = (g.scl_off + scl_bytes + 15u) & ~15u;
  const uint32_t main_end = g.gamma_off + (b_kind == B_NORM ? static_cast<uint32_t>(nk) * kel * 4u : 0u);
  const uint32_t slices_end = S > 1 ? static_cast<uint32_t>(S) * g.TS * BM * 4u : 0u;
  g.recv_off = ((main_end > slices_end ? main_end : slices_end) + 1023u) & ~1023u;
  return g;
}

// RoPE (cos, sin) rows the QKV epilogue stages: one per action position when the H positions are
// fewer than the tile's tokens, else one per token of the tile (long sequences, e.g. the prefix pass).
__host__ __device__ __forceinline__ bool rope_by_token(int H, int Nt) { return H > Nt; }

// Bytes of the epilogue stage that follows the main-loop and exchange regions: the QKV epilogue's
// RoPE (cos, sin) pairs.  (Staging the other epilogues' outputs for bulk stores was measured slower
// than direct stores: the kernel would have to wait for its stores before exiting.)
__host__ __device__ __forceinline__ uint32_t gemm_stage_bytes(int epi, int fp8, int Nt, int S, int H, int xb) {
  (void)fp8;
  (void)S;
  (void)xb;
  return epi == EPI_QKV ? static_cast<uint32_t>(rope_by_token(H, Nt) ? Nt : H) * 64u * 8u : 0u;
}

// Largest chunk count of any split-K rank: the shared-memory layout is the same in every CTA.
__host__ __device__ __forceinline__ int nk_max_of(const GemmArgs& a) { return (a.NKC + a.S - 1) / a.S; }

// Bytes of the main loop and epilogue regions; the QKV epilogue's RoPE stage ([H][64] (cos, sin)
// pairs of the m-block) follows them.
__host__ __device__ __forceinline__ uint32_t gemm_rope_off(int Nt, int stages, int b_kind, int fp8, int S, int nk,
                                                          int w4, int epi_kind, int red_tok, int kpu) {
  const GemmGeom g = gemm_geom(Nt, stages, b_kind, fp8, S, nk, w4, 1, kpu);   // kc0 odd: the larger group count
  const uint32_t kel = fp8 ? KCB : KCB / 2;
  const uint32_t main = g.gamma_off + (b_kind == B_NORM ? static_cast<uint32_t>(nk) * kel * 4u : 0u);
  const uint32_t TS = (Nt + S - 1) / S;
  // split-K slices (S > 1) or one pass of the S == 1 accumulator rows overlay the ring; the residual
  // epilogue's prefetched h rows (S > 1) follow at recv_off
  uint32_t epi = S > 1 ? static_cast<uint32_t>(S) * TS * BM * 4u : static_cast<uint32_t>(red_tok) * RED_LD * 4u;
  if (S > 1 && epi_kind == EPI_RESID && g.recv_off + 2u * TS * 64u * 4u > epi) epi = g.recv_off + 2u * TS * 64u * 4u;
  return ((main > epi ? main : epi) + 15u) & ~15u;
}

template <int EPI, int FP8, int NORM, int W4>
__global__ void __launch_bounds__(GEMM_THREADS, 2) k_gemm_tc(const __grid_constant__ GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ GemmSmem sh;
  TL_DECL
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  TL_BEGIN(10 + EPI);
  const int ks = blockIdx.x;            // split-K rank (= cluster rank)
  const int nt = blockIdx.y;            // n-tile (varies fastest after the split: CTAs that share a
  const int mb = blockIdx.z;            // weight m-block run together and read it once from HBM)
  const int Nt = a.Nt;
  const int n0 = nt * Nt;
  const int S = a.S;
  const int kc0 = ks * a.NKC / S, kc1 = (ks + 1) * a.NKC / S;
  // KPU consecutive k-chunks per ring slot (two only without B_NORM and 4-bit weights, with every
  // rank's chunk count even): one copy per operand and slot, fewer copies for the SM's copy engine
  const int KPU = (NORM || W4) ? 1 : a.kpu;
  const int nk = (kc1 - kc0) / KPU;   // ring slot fills of this CTA
  const int stages = a.stages;
  constexpr int norm = NORM;
  const int kel = FP8 ? KCB : KCB / 2;            // K elements per chunk
  const GemmGeom gm = gemm_geom(Nt, stages, NORM ? B_NORM : B_ROWS, FP8, S, nk, W4, kc0, KPU);
  const int g0 = kc0 / 2;                          // w4: first scale group of this CTA's k-range
  // ring slot addresses: B_NORM interleaves [A | B] per slot; otherwise the A slots come first and
  // the B slots follow contiguously, so that the B chunks resident before the main loop arrive in one copy
  auto a_slot = [&](int s) -> uint8_t* { return dsm + (NORM ? s * gm.slot : s * gm.a_bytes); };
  auto b_slot = [&](int s) -> uint8_t* {
    return dsm + (NORM ? s * gm.slot + gm.a_bytes : stages * gm.a_bytes + s * (gm.slot - gm.a_bytes));
  };
  float* gsm = reinterpret_cast<float*>(dsm + gm.gamma_off);

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&sh.full_a[s], W4 ? CONV_THREADS : 1);   // w4: the converters hand each chunk over
      mbar_init(&sh.raw_a[s], 1);
      mbar_init(&sh.full_b[s], norm ? CONV_THREADS : 1);
      mbar_init(&sh.empty[s], 1);
    }
    mbar_init(&sh.done, 1);
    mbar_init(&sh.hbar, 1);
    mbar_init(&sh.xbar, 1);
    mbar_init(&sh.sbar, 1);
    fence_mbar_init();
  }
  uint32_t ncols = 32;
  while (ncols < static_cast<uint32_t>(Nt)) ncols <<= 1;
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_launch();   // the next kernel may start its own prefetch now
  const uint32_t tacc = sh.tmem_base;
  // QKV: (cos, sin) of this m-block's 64 rotate-half pairs at every action position, staged while
  // the previous kernel runs (the tables are static); read by the epilogue after the main loop
  float2* rope_sh = reinterpret_cast<float2*>(dsm + gemm_rope_off(Nt, stages, NORM ? B_NORM : B_ROWS, FP8, S, nk_max_of(a), W4, EPI, a.red_tok, KPU));
  if (EPI == EPI_QKV && mb < a.MB_rot && warp >= 2) {   // warps 2-7: the producer and MMA warps go on
    const int half = a.dh >> 1;
    const bool by_tok = rope_by_token(a.H, Nt);
    for (int idx = tid - 64; idx < (by_tok ? Nt : a.H) * 64; idx += GEMM_THREADS - 64) {
      const int i = idx >> 6, p = idx & 63;
      const int j = (mb * 64 + p) % half, pos = a.P + (by_tok ? (n0 + i) % a.H : i);
      rope_sh[idx] = make_float2(a.rope_cos[pos * half + j], a.rope_sin[pos * half + j]);
    }
  }

  if (warp == 0) {
    // ---------------- bulk-copy producer
    if (lane == 0) {
      const uint8_t* wsrc = a.W + (static_cast<size_t>(mb) * a.NKC + kc0) * (BM * KCB);
      const uint32_t tb1 = static_cast<uint32_t>(Nt) * KCB;   // one k-chunk of B
      auto issue_b = [&](int i) {
        const int s = i % stages;
        uint8_t* bdst = b_slot(s);
        if (!norm) {   // B_NORM: the converters fill the slot
          mbar_arrive_expect_tx(&sh.full_b[s], KPU * tb1);
          bulk_g2s(bdst, a.act + (static_cast<size_t>(nt) * a.NKC + kc0 + i * KPU) * tb1, KPU * tb1, &sh.full_b[s]);
        }
      };
      const uint8_t* w4src = a.W + (static_cast<size_t>(mb) * a.NKC + kc0) * W4_CHUNK;
      auto issue_a = [&](int i) {
        const int s = i % stages;
        if (W4) {
          mbar_arrive_expect_tx(&sh.raw_a[s], W4_CHUNK);
          bulk_g2s(dsm + gm.rawa_off + s * W4_CHUNK, w4src + static_cast<size_t>(i) * W4_CHUNK, W4_CHUNK, &sh.raw_a[s]);
        } else {
          mbar_arrive_expect_tx(&sh.full_a[s], gm.a_bytes);
          bulk_g2s(a_slot(s), wsrc + static_cast<size_t>(i) * gm.a_bytes, gm.a_bytes, &sh.full_a[s]);
        }
      };
      const int pre = nk < stages ? nk : stages;
      if (W4) {   // the scales of this CTA's groups, one copy
        const uint32_t sb = static_cast<uint32_t>(w4_groups(kc0, nk)) * BM * 2u;
        mbar_arrive_expect_tx(&sh.sbar, sb);
        bulk_g2s(dsm + gm.scl_off, a.Wscale + (static_cast<size_t>(mb) * ((a.NKC + 1) / 2) + g0) * BM, sb, &sh.sbar);
      }
      for (int i = 0; i < pre; ++i) issue_a(i);   // weights first: they do not depend on the previous kernel
      grid_dep_wait();
      TL(1);
      if (!NORM && Nt <= 64) {   // batch-1 tiles: B chunks 0..pre-1 are contiguous in global and in shared memory: one copy
        const uint32_t tb = KPU * tb1;
        mbar_arrive_expect_tx(&sh.full_b[0], pre * tb);
        bulk_g2s(b_slot(0), a.act + (static_cast<size_t>(nt) * a.NKC + kc0) * tb1, pre * tb, &sh.full_b[0]);
        for (int i = 1; i < pre; ++i) mbar_arrive(&sh.full_b[i]);   // their first fill is covered by slot 0's copy
      } else {
        for (int i = 0; i < pre; ++i) issue_b(i);
      }
      if (S > 1 && EPI == EPI_RESID) {   // residual rows of this CTA's tokens, for the epilogue
        const int r0 = ks * Nt / S, r1 = (ks + 1) * Nt / S;
        const uint32_t rb = static_cast<uint32_t>(r1 - r0) * 256u;
        float* hst = reinterpret_cast<float*>(dsm + gm.recv_off);
        mbar_arrive_expect_tx(&sh.hbar, 2 * rb);
        for (int u = 0; u < 2; ++u)
          bulk_g2s(hst + static_cast<size_t>(u) * gm.TS * 64,
                   a.h_out + ((static_cast<size_t>(nt) * a.KB + 2 * mb + u) * Nt + r0) * 64, rb, &sh.hbar);
      }
      int issued = pre;
      for (int i = pre; i < nk; ++i) {
        const int s = i % stages;
        if (!mbar_wait(&sh.empty[s], ((i / stages) - 1) & 1, WAIT_LIMIT_NS)) {
          report_timeout(a.status, 0x100);
          break;
        }
        issue_a(i);
        issue_b(i);
        issued = i + 1;
      }
      // drain: the copies issued into this CTA's shared memory have landed before it is reused
      for (int i = (issued > stages ? issued - stages : 0); i < issued; ++i) {
        const int s = i % stages;
        const uint32_t par = (i / stages) & 1;
        if (!mbar_wait(W4 ? &sh.raw_a[s] : &sh.full_a[s], par, WAIT_LIMIT_NS) ||
            (!norm && !mbar_wait(&sh.full_b[s], par, WAIT_LIMIT_NS)))
          report_timeout(a.status, 0x101);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(FP8 ? FMT_E4M3 : FMT_BF16, BM, Nt);
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        const uint32_t par = (i / stages) & 1;
        // first pass over the ring, batch-1 tiles without B_NORM: one copy brought every resident B chunk and completes
        // slot 0; the chunks after it need no wait of their own
        const bool wait_b = NORM || Nt > 64 || i >= stages || i == 0;
        if (!mbar_wait(&sh.full_a[s], par, WAIT_LIMIT_NS) || (wait_b && !mbar_wait(&sh.full_b[s], par, WAIT_LIMIT_NS))) {
          report_timeout(a.status, 0x200);
          break;
        }
        tc_fence_after();
        if (i == 0) TL(6);
        const uint32_t a0 = smem_u32(a_slot(s)), b0 = smem_u32(b_slot(s));
        // the slot's KPU k-chunks continue the 16-byte core-matrix columns of the first (LBO apart)
        for (int k = 0; k < KPU * (KCB / 32); ++k) {
          const uint64_t ad = smem_desc(a0 + k * 2 * BM * 16, BM * 16, 128);
          const uint64_t bd = smem_desc(b0 + k * 2 * Nt * 16, Nt * 16, 128);
          if (FP8) mma_e4m3(tacc, ad, bd, idesc, (i | k) != 0);
          else mma_bf16(tacc, ad, bd, idesc, (i | k) != 0);
        }
        mma_commit(&sh.empty[s]);
      }
      mma_commit(&sh.done);
      TL(2);
    }
  } else if (norm || a.rscale || W4) {
    // ---------------- warps 2-7: per-token rstd; for B_NORM also RMSNorm(h)*gamma -> e4m3 / bf16 tile;
    // for 4-bit weights the A operand bf16(q * s) of every chunk
    const int st = tid - 64;
    // w4: chunk i's codes (slab j, row r: 8 codes in 4 B) -> bf16(q * s) in the K-major A slot
    auto convert_a = [&](int i) {
      const int s = i % stages;
      if (!mbar_wait(&sh.raw_a[s], (i / stages) & 1, WAIT_LIMIT_NS)) report_timeout(a.status, 0x310);
      const uint32_t* raw = reinterpret_cast<const uint32_t*>(dsm + gm.rawa_off + s * W4_CHUNK);
      const __nv_bfloat16* scl =
          reinterpret_cast<const __nv_bfloat16*>(dsm + gm.scl_off) + ((kc0 + i) / 2 - g0) * BM;
      uint8_t* adst = a_slot(s);
      for (int it = st; it < 8 * BM; it += CONV_THREADS) {
        const int j = it >> 7, r = it & (BM - 1);     // consecutive threads: consecutive rows
        const uint32_t wv = raw[it];
        const float sc = __bfloat162float(scl[r]);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = static_cast<float>(static_cast<int>(wv << (28 - 8 * e)) >> 28) * sc;
          const float hi = static_cast<float>(static_cast<int>(wv << (24 - 8 * e)) >> 28) * sc;
          o[e] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4*>(adst + j * (BM * 16) + (r >> 3) * 128 + (r & 7) * 16) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();   // generic-proxy writes -> visible to the tensor core
      mbar_arrive(&sh.full_a[s]);
    };
    const int pre_a = nk < stages ? nk : stages;
    if (W4) {   // static weights: convert what is resident before the dependency wait
      if (!mbar_wait(&sh.sbar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x311);
      for (int i = 0; i < pre_a; ++i) convert_a(i);
    }
    if (norm) {
      for (int idx = st; idx < nk * kel; idx += CONV_THREADS) {   // static: before the dependency wait
        const int k = kc0 * kel + idx;
        gsm[idx] = k < a.D ? a.gamma[k] : 0.f;                      // padded K: zero
      }
    }
    grid_dep_wait();
    for (int r = st; r < ((norm || a.rscale) ? Nt : 0); r += CONV_THREADS) {
      const int t = n0 + r;
      float rs = 0.f;
      if (t < a.T) {
        const float4* sp = reinterpret_cast<const float4*>(a.ssq + static_cast<size_t>(t) * a.ssq_ld);
        float4 v[4];
        const int nv = a.ssq_ld >> 2;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < nv) v[q] = sp[q];
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < nv) ss += ((v[q].x + v[q].y) + v[q].z) + v[q].w;
        rs = 1.0f / sqrtf(ss / a.D + a.eps);
      }
      sh.rstd[r] = rs;   // padded tokens become zero
    }
    conv_sync();
    if (W4)
      for (int i = pre_a; i < nk; ++i) convert_a(i);
    const float inv_sa = (norm && FP8) ? 1.0f / *a.s_a : 1.0f;
    // B_NORM (e4m3 operands): chunk i's operand tile e4m3(h * rstd * gamma / s_a) from the residual rows
    // in global memory (just written by the previous kernel, in L2), CONV_BATCH 16-feature items per
    // thread in flight; a slot is refilled once the MMAs of the chunk it held are done.
    static_assert(!NORM || FP8, "the normalising B operand is the e4m3 one");
    constexpr int CONV_BATCH = 4;
    const int jt = st & 7;   // this thread's 16-feature piece of every token row (CONV_THREADS % 8 == 0)
    for (int i = 0; i < (norm ? nk : 0); ++i) {
      const int s = i % stages;
      if (i >= stages && !mbar_wait(&sh.empty[s], ((i / stages) - 1) & 1, WAIT_LIMIT_NS)) {
        report_timeout(a.status, 0x300);
        break;
      }
      uint8_t* breg = b_slot(s);
      const int kb = (kc0 + i) * 2;   // two 64-feature blocks of h per 128-input chunk
      const float* hsrc = a.h + ((static_cast<size_t>(nt) * a.KB + kb + (jt >> 2)) * Nt) * 64 + (jt & 3) * 16;
      float4 gv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) gv[u] = *reinterpret_cast<const float4*>(gsm + i * kel + jt * 16 + 4 * u);
      for (int it0 = st; it0 < Nt * 8; it0 += CONV_BATCH * CONV_THREADS) {
        float4 hv[CONV_BATCH][4];
#pragma unroll
        for (int q = 0; q < CONV_BATCH; ++q) {
          const int it = it0 + q * CONV_THREADS;
          if (it < Nt * 8) {
            const float4* p = reinterpret_cast<const float4*>(hsrc + static_cast<size_t>(it >> 3) * 64);
#pragma unroll
            for (int u = 0; u < 4; ++u) hv[q][u] = p[u];
          }
        }
#pragma unroll
        for (int q = 0; q < CONV_BATCH; ++q) {
          const int it = it0 + q * CONV_THREADS;
          if (it < Nt * 8) {
            const int r = it >> 3;
            const float m = sh.rstd[r] * inv_sa;
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              w[u] = pack_e4m3x4(hv[q][u].x * gv[u].x * m, hv[q][u].y * gv[u].y * m, hv[q][u].z * gv[u].z * m,
                                 hv[q][u].w * gv[u].w * m);
            *reinterpret_cast<uint4*>(breg + jt * Nt * 16 + (r >> 3) * 128 + (r & 7) * 16) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      fence_proxy_async_smem();   // generic-proxy writes -> visible to the tensor core (async proxy)
      mbar_arrive(&sh.full_b[s]);
    }
  }

  // ---------------- epilogue
  grid_dep_wait();
  if (!mbar_wait(&sh.done, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x400);
  tc_fence_after();
  __syncthreads();
  if (tid == 0) TL(3);
  float* red = reinterpret_cast<float*>(dsm);   // S == 1: [red_tok][RED_LD], aliases the drained ring
  float* xs = (S > 1) ? a.xscratch + (static_cast<size_t>(nt) * a.MB + mb) * S * Nt * BM : nullptr;
  const int t_hi = min(Nt, a.T - n0);           // valid tokens of this n-tile
  // TMEM columns [cb, ce) -> red (S == 1: row stride RED_LD, from token cb) or the split-K staging
  // (S > 1: valid tokens, row stride BM) by all eight warps: warp w reads the lane quadrant w % 4;
  // warps 0-3 take the first half of the columns, warps 4-7 the rest
  auto stage_tmem = [&](int cb, int ce) {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int hc = (((ce - cb) >> 4) + 1) / 2 * 16;
    const int cbeg = cb + (warp < 4 ? 0 : hc), cend = warp < 4 ? min(cb + hc, ce) : ce;
    for (int c0 = cbeg; c0 < cend; c0 += 32) {   // up to 2 loads in flight, one wait
      uint32_t v[2][16];
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (c0 + 16 * u < cend) tmem_ld16_nowait(tacc + (static_cast<uint32_t>(q * 32) << 16) + c0 + 16 * u, v[u]);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (c0 + 16 * u < cend)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = c0 + 16 * u + j;
            if (S == 1) red[(tok - cb) * RED_LD + row] = __uint_as_float(v[u][j]);
            else if (tok < t_hi) red[tok * BM + row] = __uint_as_float(v[u][j]);   // staged for one bulk store
          }
    }
  };
  if (S > 1) {   // the partial tile (valid tokens) into the scratch with one bulk store
    stage_tmem(0, Nt);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(xs + static_cast<size_t>(ks) * Nt * BM, red, static_cast<uint32_t>(t_hi) * BM * 4u);
      bulk_commit();
      bulk_wait_all();
      fence_proxy_async_global();
    }
  }
  if (tid == 128) TL(7);
  tc_fence_before();
  const int tok0 = ks * Nt / S, tok1 = (ks + 1) * Nt / S;
  float* xst = reinterpret_cast<float*>(dsm);   // S > 1: [S][TS][128] slices of this CTA's tokens
  if (S > 1) {
    cluster_arrive_release();   // the partial tiles in scratch are visible to the cluster after this barrier
    cluster_wait_acquire();
    if (tid == 0) TL(8);
    if (tid == 0) {             // one round trip: every slice of this CTA's tokens by bulk copy
      const uint32_t sb = static_cast<uint32_t>(tok1 - tok0) * BM * 4u;
      mbar_arrive_expect_tx(&sh.xbar, S * sb);
      for (int s2 = 0; s2 < S; ++s2)
        bulk_g2s(xst + static_cast<size_t>(s2) * gm.TS * BM, xs + (static_cast<size_t>(s2) * Nt + tok0) * BM, sb,
                 &sh.xbar);
    }
    if (!mbar_wait(&sh.xbar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x500);
  }
  if (tid == 0) TL(4);

  const float al = a.alpha ? *a.alpha : 1.0f;
  int rbase = 0;   // S == 1: first token of the staged pass
  // Split-K sums of N (2 or 4) consecutive accumulator rows of one token over the cluster, in
  // rank order (deterministic), times the dequantisation / deferred-rstd scale.
  auto vals = [&](int tok, int row, float* out, auto n_tag) {
    constexpr int N = decltype(n_tag)::value;
    const float sc = a.rscale ? al * sh.rstd[tok] : al;
    float acc[N];
#pragma unroll
    for (int e = 0; e < N; ++e) acc[e] = 0.f;
    if (S == 1) {   // no split: the accumulator rows as staged (wide tiles: no per-rank predication)
      const float* p = red + (tok - rbase) * RED_LD + row;
#pragma unroll
      for (int e = 0; e < N; ++e) out[e] = p[e] * sc;
      return;
    }
    const float* p = xst + static_cast<size_t>(tok - tok0) * BM + row;
    const size_t stride = static_cast<size_t>(gm.TS) * BM;
    if (S == 2) {
#pragma unroll
      for (int e = 0; e < N; ++e) out[e] = (p[e] + p[stride + e]) * sc;   // rank order
      return;
    }
    const int ns = S;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2)
      if (s2 < ns) {
        if constexpr (N == 4) {
          const float4 v = *reinterpret_cast<const float4*>(p + s2 * stride);
          acc[0] += v.x;   // rank order
          acc[1] += v.y;
          acc[2] += v.z;
          acc[3] += v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(p + s2 * stride);
          acc[0] += v.x;
          acc[1] += v.y;
        }
      }
#pragma unroll
    for (int e = 0; e < N; ++e) out[e] = acc[e] * sc;
  };
  using Two = std::integral_constant<int, 2>;
  using Four = std::integral_constant<int, 4>;
  // Each warp takes whole tokens (tok0 + warp, + 8, ...), each lane 2 or 4 consecutive
  // features; EPU tokens per warp have their independent loads issued before any is used.
  constexpr int EPU = 4;

  // S == 1: the accumulator is staged and written in passes of red_tok tokens (a wide tile's
  // staging then fits half of an SM's shared memory and two CTAs share the SM)
  const int npass = S == 1 ? (Nt + a.red_tok - 1) / a.red_tok : 1;
  for (int pass = 0; pass < npass; ++pass) {
  const int ebeg = S == 1 ? pass * a.red_tok : tok0;
  const int eend = S == 1 ? min(Nt, ebeg + a.red_tok) : tok1;
  if (S == 1) {
    if (pass > 0) __syncthreads();   // every warp is done with the previous pass's rows
    stage_tmem(ebeg, eend);
    tc_fence_before();
    __syncthreads();
    rbase = ebeg;
  }
  if (EPI == EPI_RESID) {
    const int row = lane * 4;
    const int f = mb * BM + row;
    const bool fok = f < a.Nout;   // Nout is a multiple of 16
    const float* hst = reinterpret_cast<const float*>(dsm + gm.recv_off);   // [2][TS][64]
    if (S > 1 && !mbar_wait(&sh.hbar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x600);
    float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.xb_out && fok) g4 = *reinterpret_cast<const float4*>(a.xb_gamma + f);
    float4 gt = make_float4(1.f, 1.f, 1.f, 1.f);   // adaptive RMSNorm: gated residual update
    if (a.gate && fok) gt = *reinterpret_cast<const float4*>(a.gate + f);
    for (int tb = ebeg + warp; tb < eend; tb += 8 * EPU) {
      float4 hold[EPU];
      float acc[EPU][4];
#pragma unroll
      for (int u = 0; u < EPU; ++u) {
        const int tok = tb + 8 * u, t = n0 + tok;
        if (tok < eend && t < a.T && fok) {
          hold[u] = (S > 1) ? *reinterpret_cast<const float4*>(hst + ((row >> 6) * gm.TS + (tok - tok0)) * 64 + (row & 63))
                            : *reinterpret_cast<const float4*>(a.h_out + htile_offset_nt(nt, tok, f, Nt, a.KB));
          vals(tok, row, acc[u], Four{});
        }
      }
#pragma unroll
      for (int u = 0; u < EPU; ++u) {
        const int tok = tb + 8 * u, t = n0 + tok;
        if (tok >= eend || t >= a.T) break;   // warp-uniform
        float sq = 0.f;
        if (fok) {
          const float4 hv = make_float4(hold[u].x + gt.x * acc[u][0], hold[u].y + gt.y * acc[u][1],
                                        hold[u].z + gt.z * acc[u][2], hold[u].w + gt.w * acc[u][3]);
          sq = ((hv.x * hv.x + hv.y * hv.y) + hv.z * hv.z) + hv.w * hv.w;
          const size_t ho = htile_offset_nt(nt, tok, f, Nt, a.KB);
          if (in_bounds(a.status, ho + 3, a.ext.h, 0x9001)) *reinterpret_cast<float4*>(a.h_out + ho) = hv;
          const size_t xo = btile_offset_nt(nt, tok, 2 * f, Nt, a.NKC_x);
          if (a.xb_out && in_bounds(a.status, xo + 7, a.ext.xbuf, 0x9002))
            *reinterpret_cast<uint2*>(a.xb_out + xo) =
                make_uint2(pack_bf16x2(hv.x * g4.x, hv.y * g4.y), pack_bf16x2(hv.z * g4.z, hv.w * g4.w));
        }
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        const size_t so = static_cast<size_t>(t) * a.ssq_ld + mb;
        if (lane == 0 && in_bounds(a.status, so, a.ext.ssq, 0x9003)) a.ssq_out[so] = sq;
      }
    }
  } else if (EPI == EPI_GELU) {
    const int p = lane * 2;
    const int f = mb * 64 + p;   // F is a multiple of 64
    const float inv = (FP8 && a.s_a_out) ? 1.0f / *a.s_a_out : 1.0f;
    float2 bg = make_float2(0.f, 0.f), bu = make_float2(0.f, 0.f);   // adaptive RMSNorm shift, W b
    if (a.bias && f < a.F) {
      bg = *reinterpret_cast<const float2*>(a.bias + f);
      bu = *reinterpret_cast<const float2*>(a.bias + a.F + f);
    }
    for (int tok = ebeg + warp; tok < eend; tok += 8) {
      const int t = n0 + tok;
      if (t >= a.T || f >= a.F) break;
      float g[2], up[2];
      vals(tok, p, g, Two{});
      vals(tok, p + 64, up, Two{});
      g[0] += bg.x;
      g[1] += bg.y;
      up[0] += bu.x;
      up[1] += bu.y;
      const float u0 = gelu_tanh(g[0]) * up[0], u1 = gelu_tanh(g[1]) * up[1];
      if (FP8) {
        const size_t uo = btile_offset_nt(nt, tok, f, Nt, a.NKC_u);
        if (in_bounds(a.status, uo + 1, a.ext.ubuf, 0x9004))
          *reinterpret_cast<uint16_t*>(a.u_out + uo) =
              static_cast<uint16_t>(pack_e4m3x2(u0 * inv, u1 * inv));
      } else {
        const size_t uo = btile_offset_nt(nt, tok, 2 * f, Nt, a.NKC_u);
        if (in_bounds(a.status, uo + 3, a.ext.ubuf, 0x9004))
          *reinterpret_cast<uint32_t*>(a.u_out + uo) = pack_bf16x2(u0, u1);
      }
    }
  } else {   // EPI_QKV
    const int half = a.dh >> 1;
    if (mb < a.MB_rot) {
      const int p = lane * 2;                 // rotate-half pairs p, p+1 (same head: half is even)
      const int pi = mb * 64 + p;
      const int head = pi / half, j = pi % half;
      float2 blo = make_float2(0.f, 0.f), bhi = make_float2(0.f, 0.f);   // adaptive RMSNorm shift, W b
      if (a.bias) {
        blo = *reinterpret_cast<const float2*>(a.bias + head * a.dh + j);
        bhi = *reinterpret_cast<const float2*>(a.bias + head * a.dh + j + half);
      }
      for (int tb = ebeg + warp; tb < eend; tb += 8 * EPU) {
        float2 cs[EPU], sn[EPU];
#pragma unroll
        for (int u = 0; u < EPU; ++u) {
          const int tok = tb + 8 * u, t = n0 + tok;
          if (tok < eend && t < a.T) {
            const float4 r4 = *reinterpret_cast<const float4*>(rope_sh + (rope_by_token(a.H, Nt) ? tok : t % a.H) * 64 + p);   // pairs p, p+1
            cs[u] = make_float2(r4.x, r4.z);
            sn[u] = make_float2(r4.y, r4.w);
          }
        }
#pragma unroll
        for (int u = 0; u < EPU; ++u) {
          const int tok = tb + 8 * u, t = n0 + tok;
          if (tok >= eend || t >= a.T) break;
          const int b = t / a.H, i = t % a.H, pos = a.P + i;
          float lo[2], hi[2];
          vals(tok, p, lo, Two{});
          vals(tok, p + 64, hi, Two{});
          lo[0] += blo.x;
          lo[1] += blo.y;
          hi[0] += bhi.x;
          hi[1] += bhi.y;
          const float r00 = lo[0] * cs[u].x - hi[0] * sn[u].x, r10 = lo[0] * sn[u].x + hi[0] * cs[u].x;
          const float r01 = lo[1] * cs[u].y - hi[1] * sn[u].y, r11 = lo[1] * sn[u].y + hi[1] * cs[u].y;
          const bool isq = head < a.Hq;
          const size_t o = isq ? ((static_cast<size_t>(b) * a.Hq + head) * a.H + i) * a.dh
                               : ((static_cast<size_t>(b) * a.Hkv + (head - a.Hq)) * a.S_max + pos) * a.dh;
          __nv_bfloat16* dst = (isq ? a.q_out : a.kv_k) + o;
          if (in_bounds(a.status, o + j + half + 1, isq ? a.ext.q : a.ext.kv, isq ? 0x9005 : 0x9006)) {
            *reinterpret_cast<uint32_t*>(dst + j) = pack_bf16x2(r00, r01);
            *reinterpret_cast<uint32_t*>(dst + j + half) = pack_bf16x2(r10, r11);
          }
        }
      }
    } else {
      const int row = lane * 4;
      const int idx = (mb - a.MB_rot) * BM + row;
      const int g = idx / a.dh, d = idx % a.dh;
      float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);   // adaptive RMSNorm shift, W b
      if (a.bias) bv = *reinterpret_cast<const float4*>(a.bias + (a.Hq + a.Hkv) * a.dh + idx);
      for (int tok = ebeg + warp; tok < eend; tok += 8) {
        const int t = n0 + tok;
        if (t >= a.T) break;
        const int b = t / a.H, i = t % a.H, pos = a.P + i;
        float v4[4];
        vals(tok, row, v4, Four{});
        v4[0] += bv.x;
        v4[1] += bv.y;
        v4[2] += bv.z;
        v4[3] += bv.w;
        const size_t vo = ((static_cast<size_t>(b) * a.Hkv + g) * a.S_max + pos) * a.dh + d;
        if (in_bounds(a.status, vo + 3, a.ext.kv, 0x9007))
          *reinterpret_cast<uint2*>(a.kv_v + vo) = make_uint2(pack_bf16x2(v4[0], v4[1]), pack_bf16x2(v4[2], v4[3]));
      }
    }
  }
  }   // passes
  if (tid == 0) TL(9);
  __syncthreads();
  if (tid == 0) TL(5);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tacc, ncols);
  }
}

// ================================================================== persistent gate|up GEMM (wide tiles)
//
// One CTA per SM walks the (m-block, n-tile) tiles t = blockIdx.x, + gridDim.x, ... (consecutive t share
// the m-block, so the CTAs running together read a weight tile from HBM once).  Warp 0 lane 0 copies
// A and B chunks into the ring across tile boundaries, warp 1 lane 0 issues the MMAs into one of two
// accumulators in tensor memory, and warps 2-9 drain the other: TMEM -> shared memory in passes of
// PT_RED_TOK tokens, GeLU(gate) * up, the down projection's bf16 operand.  The epilogue of tile i thus
// runs while the MMAs of tile i + 1 do.  bf16 operands, no split-K (multi-wave shapes only).

constexpr int PT_THREADS = 320;   // warp 0: copies, warp 1: MMAs, warps 2-9: epilogue
constexpr int PT_EPI = 256;       // epilogue threads
constexpr int PT_RED_TOK = 64;    // tokens per epilogue staging pass
constexpr int PT_KPS = 2;         // k-chunks per ring slot: two large copies per slot (the copy engine of an
                                  // SM takes about a third of a microsecond per copy, one copy at a time)

struct PtSmem {
  uint64_t full_a[MAX_STAGES], full_b[MAX_STAGES], empty[MAX_STAGES];
  uint64_t tfull[2], tempty[2];   // accumulator a: MMAs done / drained by the epilogue
  uint64_t fin;                   // every MMA of the CTA done (before tensor memory is freed)
  uint32_t tmem_base;
  float rstd[NT_MAX];
};

__host__ __device__ __forceinline__ uint32_t pt_ring_bytes(int Nt, int stages) {
  return static_cast<uint32_t>(stages) * PT_KPS * (BM * KCB + static_cast<uint32_t>(Nt) * KCB);
}

__device__ __forceinline__ void pt_epi_sync() { asm volatile("bar.sync 2, 256;" ::: "memory"); }

__global__ void __launch_bounds__(PT_THREADS, 1) k_gemm_gelu_pt(const __grid_constant__ GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ PtSmem sh;
  __shared__ volatile int pt_fail;   // an epilogue wait gave up (all epilogue warps stop together)
  TL_DECL
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  TL_BEGIN(13);
  const int Nt = a.Nt, NTl = a.pt_nt, NKC = a.NKC, stages = a.stages;
  const int tiles = a.MB * NTl;
  const int my_tiles = (tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const uint32_t a_bytes = PT_KPS * BM * KCB, b_bytes = PT_KPS * static_cast<uint32_t>(Nt) * KCB;   // per slot
  const int NSC = NKC / PT_KPS;   // slots of one tile (NKC is a multiple of PT_KPS)
  auto a_slot = [&](int s) { return dsm + s * a_bytes; };
  auto b_slot = [&](int s) { return dsm + stages * a_bytes + s * b_bytes; };
  float* red = reinterpret_cast<float*>(dsm + pt_ring_bytes(Nt, stages));   // [PT_RED_TOK][RED_LD]
  auto tile_of = [&](int i, int& mb, int& nt) {
    const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    mb = t / NTl;
    nt = t - mb * NTl;
  };

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&sh.full_a[s], 1);
      mbar_init(&sh.full_b[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.tfull[i], 1);
      mbar_init(&sh.tempty[i], PT_EPI);
    }
    mbar_init(&sh.fin, 1);
    pt_fail = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_launch();
  const uint32_t tbase = sh.tmem_base;
  const int total = my_tiles * NSC;   // ring slots this CTA fills

  if (warp == 0) {
    // ---------------- copies: slot fill q holds k-chunks PT_KPS * (q % NSC) .. of this CTA's tile q / NSC
    if (lane == 0) {
      auto issue_a = [&](int q) {
        int mb, nt;
        tile_of(q / NSC, mb, nt);
        const int s = q % stages;
        mbar_arrive_expect_tx(&sh.full_a[s], a_bytes);
        bulk_g2s(a_slot(s), a.W + (static_cast<size_t>(mb) * NSC + q % NSC) * a_bytes, a_bytes, &sh.full_a[s]);
      };
      auto issue_b = [&](int q) {
        int mb, nt;
        tile_of(q / NSC, mb, nt);
        const int s = q % stages;
        mbar_arrive_expect_tx(&sh.full_b[s], b_bytes);
        bulk_g2s(b_slot(s), a.act + (static_cast<size_t>(nt) * NSC + q % NSC) * b_bytes, b_bytes, &sh.full_b[s]);
      };
      const int pre = total < stages ? total : stages;
      for (int q = 0; q < pre; ++q) issue_a(q);   // weights do not depend on the previous kernel
      grid_dep_wait();
      TL(1);
      for (int q = 0; q < pre; ++q) issue_b(q);
      int issued = pre;
      for (int q = pre; q < total; ++q) {
        const int s = q % stages;
        if (!mbar_wait(&sh.empty[s], ((q / stages) - 1) & 1, WAIT_LIMIT_NS)) {
          report_timeout(a.status, 0xB100);
          break;
        }
        issue_a(q);
        issue_b(q);
        issued = q + 1;
      }
      // drain: every copy issued into this CTA's shared memory has landed before the CTA exits
      for (int q = (issued > stages ? issued - stages : 0); q < issued; ++q) {
        const int s = q % stages;
        const uint32_t par = (q / stages) & 1;
        if (!mbar_wait(&sh.full_a[s], par, WAIT_LIMIT_NS) || !mbar_wait(&sh.full_b[s], par, WAIT_LIMIT_NS))
          report_timeout(a.status, 0xB101);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMAs: tile i into accumulator i & 1 once the epilogue has drained it (tile i - 2)
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(FMT_BF16, BM, Nt);
      int q = 0;
      bool ok = true;
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int acc = i & 1;
        if (i >= 2 && !mbar_wait(&sh.tempty[acc], ((i >> 1) - 1) & 1, WAIT_LIMIT_NS)) {
          report_timeout(a.status, 0xB200);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tacc = tbase + static_cast<uint32_t>(acc) * 256u;
        for (int c = 0; c < NSC; ++c, ++q) {
          const int s = q % stages;
          const uint32_t par = (q / stages) & 1;
          if (!mbar_wait(&sh.full_a[s], par, WAIT_LIMIT_NS) || !mbar_wait(&sh.full_b[s], par, WAIT_LIMIT_NS)) {
            report_timeout(a.status, 0xB201);
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c2 = 0; c2 < PT_KPS; ++c2) {   // the slot's k-chunks, each a [rows x 128 B] operand tile
            const uint32_t a0 = smem_u32(a_slot(s) + c2 * BM * KCB), b0 = smem_u32(b_slot(s) + c2 * Nt * KCB);
#pragma unroll
            for (int k = 0; k < KCB / 32; ++k)
              mma_bf16(tacc, smem_desc(a0 + k * 2 * BM * 16, BM * 16, 128), smem_desc(b0 + k * 2 * Nt * 16, Nt * 16, 128),
                       idesc, (c | c2 | k) != 0);
          }
          mma_commit(&sh.empty[s]);
        }
        if (ok) mma_commit(&sh.tfull[acc]);
      }
      // every MMA issued has completed before the accumulators are freed, also when a wait gave up and
      // no tile commit tracks the last ones (on the normal path the epilogue has waited for them already)
      mma_commit(&sh.fin);
      if (!mbar_wait(&sh.fin, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0xB202);
    }
  } else {
    // ---------------- epilogue (warps 2-9; warp w reads the TMEM lane quadrant w % 4, warps 2-5 the
    // first half of a pass's token columns, warps 6-9 the rest; each warp then takes whole tokens,
    // each lane two consecutive gate/up feature pairs)
    const int ew = warp - 2, etid = tid - 64;
    const int q4 = warp & 3, row = q4 * 32 + lane;
    const int p = lane * 2;
    grid_dep_wait();   // the Σh² partials and the operand buffer belong to the previous kernels
    const float al = a.alpha ? *a.alpha : 1.0f;
    for (int i = 0; i < my_tiles; ++i) {
      const int acc = i & 1;
      int mb, nt;
      tile_of(i, mb, nt);
      const int n0 = nt * Nt;
      const uint32_t tacc = tbase + static_cast<uint32_t>(acc) * 256u;
      if (!mbar_wait(&sh.tfull[acc], (i >> 1) & 1, WAIT_LIMIT_NS)) pt_fail = 1;   // MMAs of tile i done
      pt_epi_sync();   // the previous tile's reads of rstd and of the staged rows are done; pt_fail agreed
      if (pt_fail) {
        if (etid == 0) report_timeout(a.status, 0xB300);
        break;
      }
      if (a.rscale)
        for (int r = etid; r < Nt; r += PT_EPI) {
          const int t = n0 + r;
          float rs = 0.f;
          if (t < a.T) {
            const float4* sp = reinterpret_cast<const float4*>(a.ssq + static_cast<size_t>(t) * a.ssq_ld);
            float4 v[4];
            const int nv = a.ssq_ld >> 2;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
              if (qq < nv) v[qq] = sp[qq];
            float ss = 0.f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
              if (qq < nv) ss += ((v[qq].x + v[qq].y) + v[qq].z) + v[qq].w;
            rs = 1.0f / sqrtf(ss / a.D + a.eps);
          }
          sh.rstd[r] = rs;   // padded tokens become zero
        }
      tc_fence_after();
      const int f = mb * 64 + p;   // F is a multiple of 64
      float2 bg = make_float2(0.f, 0.f), bu = make_float2(0.f, 0.f);   // adaptive RMSNorm shift, W b
      if (a.bias) {
        bg = *reinterpret_cast<const float2*>(a.bias + f);
        bu = *reinterpret_cast<const float2*>(a.bias + a.F + f);
      }
      for (int cb = 0; cb < Nt; cb += PT_RED_TOK) {
        const int ce = min(Nt, cb + PT_RED_TOK);
        if (cb > 0) pt_epi_sync();   // the previous pass's staged rows have been read
        {
          const int hc = (((ce - cb) >> 4) + 1) / 2 * 16;
          const int cbeg = cb + (ew < 4 ? 0 : hc), cend = ew < 4 ? min(cb + hc, ce) : ce;
          for (int c0 = cbeg; c0 < cend; c0 += 32) {   // up to 2 loads in flight, one wait
            uint32_t v[2][16];
#pragma unroll
            for (int u = 0; u < 2; ++u)
              if (c0 + 16 * u < cend) tmem_ld16_nowait(tacc + (static_cast<uint32_t>(q4 * 32) << 16) + c0 + 16 * u, v[u]);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u)
              if (c0 + 16 * u < cend)
#pragma unroll
                for (int j = 0; j < 16; ++j) red[(c0 + 16 * u + j - cb) * RED_LD + row] = __uint_as_float(v[u][j]);
          }
        }
        if (ce == Nt) {   // the accumulator is drained: the MMAs of tile i + 2 may use it
          tc_fence_before();
          mbar_arrive(&sh.tempty[acc]);
        }
        pt_epi_sync();   // this pass's rows are staged
        for (int tok = cb + ew; tok < ce; tok += 8) {
          const int t = n0 + tok;
          if (t >= a.T) break;
          const float sc = a.rscale ? al * sh.rstd[tok] : al;
          const float* rr = red + (tok - cb) * RED_LD;
          const float g0 = rr[p] * sc + bg.x, g1 = rr[p + 1] * sc + bg.y;
          const float u0 = rr[p + 64] * sc + bu.x, u1 = rr[p + 65] * sc + bu.y;
          const size_t uo = btile_offset_nt(nt, tok, 2 * f, Nt, a.NKC_u);
          if (in_bounds(a.status, uo + 3, a.ext.ubuf, 0x9004))
            *reinterpret_cast<uint32_t*>(a.u_out + uo) = pack_bf16x2(gelu_tanh(g0) * u0, gelu_tanh(g1) * u1);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ================================================================== attention

struct AttnGeom {
  uint32_t q_bytes, kv_bytes, obuf_bytes, recv_off, rowb;
  int R;   // rows per owner (max)
};

__host__ __device__ __forceinline__ AttnGeom attn_geom(int H, int dh, int KC, int C) {
  AttnGeom g;
  const int Hp = (H + 15) & ~15;
  const int LD = dh + ATT_PAD;
  g.q_bytes = static_cast<uint32_t>(Hp) * LD * 2;
  g.kv_bytes = 2u * static_cast<uint32_t>(KC) * LD * 2;
  g.rowb = static_cast<uint32_t>(dh + 4) * 4;                  // O row + (max, sum) + pad
  g.obuf_bytes = static_cast<uint32_t>(Hp) * g.rowb;          // partial rows of this chunk, overlays Q/K/V
  g.recv_off = 0;
  g.R = (H + C - 1) / C;
  return g;
}

template <int DH>
__global__ void __launch_bounds__(256) k_attn_tc(const __grid_constant__ AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ uint64_t stage_bar;
  __shared__ float w_sh[16][128];   // merge weight of chunk s for owned row rr (C <= 16, rows <= H <= 128)
  __shared__ float inv_den[128];
  TL_DECL
  TL_BEGIN(20);
  constexpr int LD = DH + ATT_PAD;       // bf16 row stride in shared memory
  constexpr int OLD = DH + 4;            // fp32 row stride of the partial-O rows
  const int c = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const int g = (j * a.Hkv) / a.Hq;      // consecutive query-head groups share a KV head
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, Hp = (H + 15) & ~15;
  const int S = a.P + H;
  const int C = a.C;
  const int key0 = c * a.KC;
  const int nkeys = min(a.KC, S - key0);
  const AttnGeom gm = attn_geom(H, DH, a.KC, C);
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(dsm);
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(dsm + gm.q_bytes);
  __nv_bfloat16* Vs = Ks + a.KC * LD;
  float* Obuf = reinterpret_cast<float*>(dsm);                  // C == 1, after compute: [Hp][OLD]
  // C > 1: this CTA's partial rows in the L2 scratch, [C][H][OLD] per (sample, head)
  float* xs = (C > 1) ? a.xscratch + (static_cast<size_t>(b) * a.Hq + j) * C * H * OLD : nullptr;
  const __nv_bfloat16* kg = a.kv_k + ((static_cast<size_t>(b) * a.Hkv + g) * a.S_max) * DH;
  const __nv_bfloat16* vg = a.kv_v + ((static_cast<size_t>(b) * a.Hkv + g) * a.S_max) * DH;
  constexpr int VPR = DH / 8;            // 16-byte vectors per row
  if (tid == 0) {
    mbar_init(&stage_bar, 1);
    fence_mbar_init();
  }
  grid_dep_launch();
  // prefix keys/values do not depend on the previous kernel: start their loads first
  for (int it = tid; it < a.KC * VPR; it += blockDim.x) {
    const int r = it / VPR, v = it % VPR;
    const int key = key0 + r;
    if (key < a.P || r >= nkeys) {
      const bool ok = r < nkeys;
      cp_async16(Ks + r * LD + v * 8, kg + static_cast<size_t>(ok ? key : 0) * DH + v * 8, ok);
      cp_async16(Vs + r * LD + v * 8, vg + static_cast<size_t>(ok ? key : 0) * DH + v * 8, ok);
    }
  }
  cp_async_commit();
  grid_dep_wait();
  if (tid == 0) TL(1);
  for (int it = tid; it < a.KC * VPR; it += blockDim.x) {
    const int r = it / VPR, v = it % VPR;
    const int key = key0 + r;
    if (key >= a.P && r < nkeys) {
      cp_async16(Ks + r * LD + v * 8, kg + static_cast<size_t>(key) * DH + v * 8, true);
      cp_async16(Vs + r * LD + v * 8, vg + static_cast<size_t>(key) * DH + v * 8, true);
    }
  }
  const __nv_bfloat16* qg = a.q + ((static_cast<size_t>(b) * a.Hq + j) * H) * DH;
  for (int it = tid; it < Hp * VPR; it += blockDim.x) {
    const int r = it / VPR, v = it % VPR;
    cp_async16(Qs + r * LD + v * 8, qg + static_cast<size_t>(r < H ? r : 0) * DH + v * 8, r < H);
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
  if (tid == 0) TL(2);

  const int gq = lane >> 2, tq = lane & 3;
  const float sl2 = a.scale * 1.4426950408889634f;   // scores in log2 units
  const int n_rg = Hp / 16;                           // one pass: n_rg <= number of warps
  const int rg = warp;
  const bool active = rg < n_rg;
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
      for (int n = 0; n < ATTN_SUBK / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = kb + n * 8 + tq * 2 + (e & 1);
          float v = sacc[n][e] * sl2;
          if (key >= nkeys) v = -INFINITY;
          sacc[n][e] = v;
          mnew[e >> 1] = fmaxf(mnew[e >> 1], v);
        }
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
      for (int n = 0; n < ATTN_SUBK / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = exp2f(sacc[n][e] - mnew[e >> 1]);
          sacc[n][e] = p;
          psum[e >> 1] += p;
        }
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
  if (C > 1) {
    // partial rows staged in shared memory (over the dead Q/K/V), one bulk store into the
    // scratch, then one cluster barrier
    __syncthreads();   // every warp is done with Q/K/V
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
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(xs + static_cast<size_t>(c) * H * OLD, Obuf, static_cast<uint32_t>(H) * OLD * 4u);
      bulk_commit();
      bulk_wait_all();
      fence_proxy_async_global();
      TL(3);
    }
    cluster_arrive_release();
    cluster_wait_acquire();
    if (tid == 0) TL(6);
  } else {
    __syncthreads();   // every warp is done with Q/K/V before the partial rows overwrite them
    if (tid == 0) TL(3);
    if (active) {
      const int r0 = rg * 16 + gq;
#pragma unroll
      for (int n = 0; n < DH / 8; ++n) {
        const int col = n * 8 + tq * 2;
        Obuf[r0 * OLD + col] = oacc[n][0];
        Obuf[r0 * OLD + col + 1] = oacc[n][1];
        Obuf[(r0 + 8) * OLD + col] = oacc[n][2];
        Obuf[(r0 + 8) * OLD + col + 1] = oacc[n][3];
      }
      if (tq == 0) {
        Obuf[r0 * OLD + DH] = mrow[0];
        Obuf[r0 * OLD + DH + 1] = lrow[0];
        Obuf[(r0 + 8) * OLD + DH] = mrow[1];
        Obuf[(r0 + 8) * OLD + DH + 1] = lrow[1];
      }
    }
    __syncthreads();
  }
  // ---------------- merge the rows this CTA owns over the key chunks, in rank order
  const int r_lo = c * H / C, r_hi = (c + 1) * H / C;
  // row rr (relative to r_lo) of chunk s: src + (s * sstride + r_lo + rr) * OLD
  // C > 1: one round trip brings this CTA's rows of every chunk into shared memory, [C][R][OLD]
  float* stage = reinterpret_cast<float*>(dsm);
  if (C > 1) {
    if (tid == 0) {
      const uint32_t sb = static_cast<uint32_t>(r_hi - r_lo) * gm.rowb;
      mbar_arrive_expect_tx(&stage_bar, C * sb);
      if (sb)
        for (int s2 = 0; s2 < C; ++s2)
          bulk_g2s(stage + static_cast<size_t>(s2) * gm.R * OLD, xs + (static_cast<size_t>(s2) * H + r_lo) * OLD, sb,
                   &stage_bar);
    }
    if (!mbar_wait(&stage_bar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x704);
  }
  // row rr of chunk s: src + (s * sstride + roff + rr) * OLD
  const float* src = (C > 1) ? stage : Obuf;
  const size_t sstride = (C > 1) ? static_cast<size_t>(gm.R) : 0;
  const int roff = (C > 1) ? 0 : r_lo;
  auto ld2 = [&](const float* p) -> float2 { return *reinterpret_cast<const float2*>(p); };
  if (tid == 0) TL(4);
  const int nr = r_hi - r_lo;
  if (tid < nr) {
    float mv[16], lv[16];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      if (s < C) {
        const float2 ml = ld2(src + (s * sstride + roff + tid) * OLD + DH);
        mv[s] = ml.x;
        lv[s] = ml.y;
      } else {
        mv[s] = -INFINITY;
        lv[s] = 0.f;
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < 16; ++s) M = fmaxf(M, mv[s]);
    float den = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      if (s < C) {
        const float e = exp2f(mv[s] - M);
        w_sh[s][tid] = e;
        den += e * lv[s];
      }
    }
    inv_den[tid] = 1.0f / den;
  }
  __syncthreads();
  if (tid == 0) TL(7);
  const float inv_sa = (a.fp8 && a.s_a) ? 1.0f / *a.s_a : 1.0f;
  // eight consecutive features per work item: one 16-byte (bf16) or 8-byte (e4m3) store
  for (int it = tid; it < nr * (DH / 8); it += blockDim.x) {
    const int rr = it / (DH / 8), d0 = (it % (DH / 8)) * 8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s)
      if (s < C) {
        const float w = w_sh[s][rr];
        const float* p = src + (s * sstride + roff + rr) * OLD + d0;
        const float4 v0 = *reinterpret_cast<const float4*>(p), v1 = *reinterpret_cast<const float4*>(p + 4);
        acc[0] += w * v0.x;   // rank order
        acc[1] += w * v0.y;
        acc[2] += w * v0.z;
        acc[3] += w * v0.w;
        acc[4] += w * v1.x;
        acc[5] += w * v1.y;
        acc[6] += w * v1.z;
        acc[7] += w * v1.w;
      }
    const float id = inv_den[rr];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= id;
    const int t = b * H + r_lo + rr;
    const int kidx = j * DH + d0;
    const size_t ob = a.o_rowmajor ? (static_cast<size_t>(t) * a.Hq * DH + kidx) * 2
                    : a.fp8 ? btile_offset(t, kidx, a.Nt, a.NKC_o) : btile_offset(t, 2 * kidx, a.Nt, a.NKC_o);
    if (!in_bounds(a.status, ob + (a.fp8 && !a.o_rowmajor ? 7 : 15), a.o_extent, 0x9010)) continue;
    if (a.o_rowmajor) {
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(t) * a.Hq * DH + kidx) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                     pack_bf16x2(acc[6], acc[7]));
    } else if (a.fp8) {
      *reinterpret_cast<uint2*>(a.o + btile_offset(t, kidx, a.Nt, a.NKC_o)) =
          make_uint2(pack_e4m3x4(acc[0] * inv_sa, acc[1] * inv_sa, acc[2] * inv_sa, acc[3] * inv_sa),
                     pack_e4m3x4(acc[4] * inv_sa, acc[5] * inv_sa, acc[6] * inv_sa, acc[7] * inv_sa));
    } else {
      *reinterpret_cast<uint4*>(a.o + btile_offset(t, 2 * kidx, a.Nt, a.NKC_o)) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                     pack_bf16x2(acc[6], acc[7]));
    }
  }
  __syncthreads();
  if (tid == 0) TL(5);
}

// ================================================================== attention on tcgen05
//
// One CTA per (sample b, KV head g, tile of 128 query rows, key chunk c); the rows of a tile
// are the (query head, action row) pairs of every query head that reads KV head g, so the
// chunk's K and V are staged once for the whole group.  Per 64-key sub-chunk:
//   K, V               tensor-map copies (128-byte swizzle) by one thread of a copy / MMA warp
//   S = Q K^T          tcgen05 (M = 128 rows, N = 64 keys, K = dh), fp32 in tensor memory
//   online softmax     two threads per row: S row from tensor memory, running max / sum,
//                      P = 2^(s - m) in bf16 into shared memory, O rescaled in tensor memory
//   O += P V           tcgen05 (M = 128, N = dh, K = 64 keys), V read MN-major as stored
// The softmax warps and the copy / MMA thread hand sub-chunks over through mbarriers only.
// Chunks (a cluster when C > 1) are merged over (O, max, sum) rows in the L2 scratch with the
// same rank-order log-sum-exp weights as the flash-decoding merge.

constexpr int UA_SUB = 64;        // keys per sub-chunk
constexpr float UA_RESCALE = 8.f; // the softmax reference moves when the row maximum grows by more (log2 units)
constexpr int UA_SOFTMAX = 256;   // softmax threads, two per query row of the tile: warps w and w + 4 share
                                  // the row's lane quadrant of tensor memory, each takes half of the keys'
                                  // exponentials and half of the O columns
constexpr int UA_THREADS = UA_SOFTMAX + 32;   // + one warp whose lane 0 issues the copies and the MMAs

struct UAttnGeom {
  uint32_t q_off, k_off0, k_off1, v_off0, v_off1, p_off0, p_off1, w_off, total, tcols, o_col;
};

// Shared memory: Q tile, two K and two V sub-chunk buffers, two P tiles.  Tensor memory: the
// scores of two sub-chunks at columns 0 and UA_SUB, O at o_col.  The merge stage of the split-KV
// case (at most 144 rows of dh + 4 floats) and the merge weights after it overlay the buffers.
__host__ __device__ __forceinline__ UAttnGeom uattn_geom(int dh) {
  UAttnGeom g;
  const uint32_t q = 128u * dh * 2u, kv = static_cast<uint32_t>(UA_SUB) * dh * 2u, pt = 128u * UA_SUB * 2u;
  g.q_off = 0;
  g.k_off0 = q;
  g.v_off0 = q + kv;
  g.k_off1 = q + 2 * kv;
  g.v_off1 = q + 3 * kv;
  g.p_off0 = q + 4 * kv;
  g.p_off1 = g.p_off0 + pt;
  g.total = g.p_off1 + pt;
  g.w_off = 144u * (dh + 4) * 4u;
  g.tcols = dh == 256 ? 512u : 256u;
  g.o_col = dh == 256 ? 256u : 128u;
  return g;
}

template <int DH>
__global__ void __launch_bounds__(UA_THREADS, 1) k_attn_umma(const __grid_constant__ AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ uint64_t bar_s[2], bar_o[2], bar_p[2], kfull[2], vfull[2], stage_bar, fin_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;             // a wait gave up: the other role stops waiting too
  __shared__ float inv_den[128];
  __shared__ float l_sh[2][128];         // the two halves' softmax sums of each row
  TL_DECL
  TL_BEGIN(20);
  constexpr int OLD = DH + 4;            // fp32 row stride of the partial-O rows
  constexpr int VPR = DH / 8;            // 16-byte vectors per Q row
  constexpr int NBX = DH / 64;           // 64-feature boxes (128-byte rows) per K or V sub-chunk
  constexpr uint32_t IDESC_S = idesc_f32acc(FMT_BF16, 128, UA_SUB);
  constexpr uint32_t IDESC_O = idesc_f32acc(FMT_BF16, 128, DH) | IDESC_B_MN_MAJOR;
  const UAttnGeom gm = uattn_geom(DH);
  const int c = blockIdx.x, y = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool sm_thread = tid < UA_SOFTMAX;        // softmax warps 0-7: two threads per query row
  const bool mma_thread = tid == UA_SOFTMAX;      // warp 8, lane 0: tensor-map copies and MMAs
  const int row = tid & 127, hh = (tid >> 7) & 1; // a softmax thread's row of the tile and half
  const int G = a.Hq / a.Hkv;            // query heads per KV head (consecutive heads)
  const int R = G * a.H;                 // query rows of one KV group
  const int MT = (R + 127) >> 7;
  const int g = y / MT, row0 = (y - g * MT) * 128;
  const int Rv = min(128, R - row0);     // valid rows of this tile
  const int S = a.P + a.H;
  const int C = a.C;
  const int key0 = c * a.KC;
  const int nkeys = min(a.KC, S - key0);
  const int nsub = (nkeys + UA_SUB - 1) / UA_SUB;
  const int zkv = b * a.Hkv + g;         // K/V tensor-map plane of (sample, KV head)
  // the group's query rows are contiguous: heads g*G.. of sample b, H rows each
  const __nv_bfloat16* qg = a.q + ((static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G) * a.H + row0) * DH;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_o[i], 1);
      mbar_init(&bar_p[i], UA_SOFTMAX);
      mbar_init(&kfull[i], 1);
      mbar_init(&vfull[i], 1);
    }
    mbar_init(&stage_bar, 1);
    mbar_init(&fin_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, gm.tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_launch();
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tS = tmem_base, tO = tmem_base + gm.o_col;
  auto Kbuf = [&](int bf) { return dsm + (bf ? gm.k_off1 : gm.k_off0); };
  auto Vbuf = [&](int bf) { return dsm + (bf ? gm.v_off1 : gm.v_off0); };
  auto Pbuf = [&](int bf) { return dsm + (bf ? gm.p_off1 : gm.p_off0); };
  volatile int* abort_v = &abort_flag;

  // K or V of sub-chunk j by tensor map (the MMA thread): NBX boxes of 64 keys x 64 features, each
  // 64 rows of 128 bytes swizzled in 1 KB atoms, 8 KB apart.  Keys past the sequence read as zeros;
  // keys past this chunk are real keys, masked in the softmax.
  int k_issued = 0, v_issued = 0;
  auto load_kv = [&](const CUtensorMap* tm, uint8_t* dst, uint64_t* bar, int j) {
    mbar_arrive_expect_tx(bar, UA_SUB * DH * 2);
    if (a.kv_boxes == 1) tma_load_4d(dst, tm, 0, key0 + j * UA_SUB, 0, zkv, bar);   // [feature block][key][128 B]
    else
      for (int x = 0; x < NBX; ++x) tma_load_3d(dst + x * (UA_SUB * 128), tm, x * 64, key0 + j * UA_SUB, zkv, bar);
  };
  auto load_k = [&](int j) {
    load_kv(&a.tm_k, Kbuf(j & 1), &kfull[j & 1], j);
    k_issued = j + 1;
  };
  auto load_v = [&](int j) {
    load_kv(&a.tm_v, Vbuf(j & 1), &vfull[j & 1], j);
    v_issued = j + 1;
  };
  // a sub-chunk whose 64 keys all precede the action rows does not depend on the previous kernel
  auto prefix_only = [&](int j) { return key0 + (j + 1) * UA_SUB <= a.P; };
  const int npro = nsub < 2 ? nsub : 2;
  if (mma_thread)
    for (int j = 0; j < npro; ++j)
      if (prefix_only(j)) {
        load_k(j);
        load_v(j);
      }
  grid_dep_wait();
  if (tid == 0) TL(1);
  if (mma_thread)
    for (int j = 0; j < npro; ++j)
      if (!prefix_only(j)) {
        load_k(j);
        load_v(j);
      }
  if (sm_thread) {   // Q tile, K-major [16-byte column][128 rows][16 B]: the two threads of a row copy half each
    const bool qv = row < Rv;
    uint8_t* dst = dsm + gm.q_off + row * 16 + hh * (VPR / 2) * 2048;
    const __nv_bfloat16* src = qg + static_cast<size_t>(qv ? row : 0) * DH + hh * (VPR / 2) * 8;
#pragma unroll
    for (int j = 0; j < VPR / 2; ++j) cp_async16(dst + j * 2048, src + j * 8, qv);
    cp_async_commit();
    cp_async_wait_all();
    fence_proxy_async_smem();   // cp.async writes -> visible to the tensor core
  }
  __syncthreads();   // Q in place
  if (tid == 0) TL(2);

  bool ok = true;
  float m_run = -INFINITY, l_run = 0.f;
  if (mma_thread) {
    // ---------------- copies and MMAs.  Per sub-chunk sc: K(sc+2) once S(sc) is done; O += P(sc) V(sc)
    // once the softmax of sc has arrived; S(sc+2) into the score buffer that softmax just read; V(sc+2)
    // once O(sc) is done.  The tensor core thus computes S(sc+1) while the softmax of sc runs.
    auto issue_s = [&](int j) {   // S(j) = Q K(j)^T into score buffer j & 1 once K(j) has landed
      if (!mbar_wait(&kfull[j & 1], (j >> 1) & 1, WAIT_LIMIT_NS)) return false;
      tc_fence_after();
      const uint32_t qa = smem_u32(dsm + gm.q_off), ka = smem_u32(Kbuf(j & 1));
#pragma unroll
      for (int k = 0; k < DH / 16; ++k)
        mma_bf16(tS + (j & 1) * UA_SUB, smem_desc(qa + k * 2 * 2048, 2048, 128),
                 smem_desc_sw128(ka + (k >> 2) * (UA_SUB * 128) + (k & 3) * 32, 16, 1024), IDESC_S, k > 0);
      mma_commit(&bar_s[j & 1]);
      return true;
    };
    ok = issue_s(0) && (nsub < 2 || issue_s(1));
    for (int sc = 0; ok && sc < nsub; ++sc) {
      const int bf = sc & 1;
      if (sc + 2 < nsub) {
        ok = mbar_wait(&bar_s[bf], (sc >> 1) & 1, WAIT_LIMIT_NS) && !*abort_v;
        if (!ok) break;
        load_k(sc + 2);
      }
      ok = mbar_wait(&bar_p[bf], (sc >> 1) & 1, WAIT_LIMIT_NS) && mbar_wait(&vfull[bf], (sc >> 1) & 1, WAIT_LIMIT_NS) &&
           !*abort_v;
      if (!ok) break;
      tc_fence_after();
      const uint32_t pa = smem_u32(Pbuf(bf)), va = smem_u32(Vbuf(bf));
#pragma unroll
      for (int k = 0; k < UA_SUB / 16; ++k)
        mma_bf16(tO, smem_desc(pa + k * 2 * 2048, 2048, 128), smem_desc_sw128(va + k * 2 * 1024, UA_SUB * 128, 1024),
                 IDESC_O, (sc > 0 || k > 0) ? 1u : 0u);
      mma_commit(&bar_o[bf]);
      if (sc + 2 < nsub) {
        ok = issue_s(sc + 2) && mbar_wait(&bar_o[bf], (sc >> 1) & 1, WAIT_LIMIT_NS);
        if (!ok) break;
        load_v(sc + 2);
      }
    }
    if (!ok) {
      *abort_v = 1;
      report_timeout(a.status, 0x700);
    }
    // every MMA issued has completed before tensor memory is read back or freed, also after a give-up
    // (on the normal path the softmax threads wait for the last O += P V as well)
    mma_commit(&fin_bar);
    if (!mbar_wait(&fin_bar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x705);
  } else if (sm_thread) {
    // ---------------- online softmax (two threads per row, each half of the keys' exponentials)
    const float sl2 = a.scale * 1.4426950408889634f;   // scores in log2 units
    for (int sc = 0; sc < nsub; ++sc) {
      const int bf = sc & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_s[bf], (sc >> 1) & 1, WAIT_LIMIT_NS) && !*abort_v)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[UA_SUB];
#pragma unroll
      for (int u = 0; u < UA_SUB / 16; ++u) tmem_ld16_nowait(tS + bf * UA_SUB + lane_base + 16 * u, sv + 16 * u);
      tmem_wait_ld();
      const int kb = sc * UA_SUB;
      // both threads of a row take the maximum over all 64 raw scores (four independent chains); the
      // scale sl2 > 0 is applied after it
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (kb + UA_SUB > nkeys) {   // the chunk's last sub-chunk: keys past it do not count
#pragma unroll
        for (int jj = 0; jj < UA_SUB; ++jj)
          if (kb + jj >= nkeys) sv[jj] = __float_as_uint(-INFINITY);
      }
#pragma unroll
      for (int jj = 0; jj < UA_SUB; ++jj) mq[jj & 3] = fmaxf(mq[jj & 3], __uint_as_float(sv[jj]));
      const float mx = fmaxf(m_run, fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * sl2);   // log2 units
      // The reference of the exponentials moves only when the row maximum has grown by more than
      // UA_RESCALE (log2 units): P stays below 2^UA_RESCALE, the sum and O are relative to the same
      // reference, and O / l is unchanged; O in tensor memory is rescaled only when a row's reference
      // moves, which after the first sub-chunks is rare.
      const float ref = (mx > m_run + UA_RESCALE) ? mx : m_run;
      const float corr = exp2f(m_run - ref);
      const bool resc = sc > 0 && __any_sync(0xffffffffu, corr != 1.f);
      // P buffer bf was read by O += P V of sub-chunk sc - 2
      if (sc >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar_o[bf], ((sc - 2) >> 1) & 1, WAIT_LIMIT_NS))) {
        ok = false;
        break;
      }
      // this thread writes keys 32*hh .. 32*hh + 31 of its row: 2^(s*sl2 - ref) in bf16
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint8_t* prow = Pbuf(bf) + (row >> 3) * 128 + (row & 7) * 16;   // K-major [128 x 64]
      auto expo = [&](auto half) {   // compile-time key range, so that sv stays in registers
        constexpr int K0 = decltype(half)::value * (UA_SUB / 2);
#pragma unroll
        for (int k2 = 0; k2 < UA_SUB / 16; ++k2) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2_approx(fmaf(__uint_as_float(sv[K0 + k2 * 8 + e]), sl2, -ref));
            ps[e & 3] += p[e];
          }
          *reinterpret_cast<uint4*>(prow + (K0 / 8 + k2) * 2048) = make_uint4(
              pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
        }
      };
      if (hh == 0) expo(std::integral_constant<int, 0>{});   // warp-uniform
      else expo(std::integral_constant<int, 1>{});
      l_run = l_run * corr + ((ps[0] + ps[1]) + (ps[2] + ps[3]));   // this half's keys
      m_run = ref;
      if (resc) {   // O(sc-1) complete before this warp's rows of O are rescaled
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_o[bf ^ 1], ((sc - 1) >> 1) & 1, WAIT_LIMIT_NS))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = hh * (DH / 2); c0 < (hh + 1) * (DH / 2); c0 += 16) {   // this thread's half of O
          uint32_t ov[16];
          tmem_ld16_nowait(tO + lane_base + c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
          tmem_st16(tO + lane_base + c0, ov);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();   // P (generic-proxy stores) -> visible to the tensor core
      tc_fence_before();          // S read and O rescaled before the MMA thread moves on
      mbar_arrive(&bar_p[bf]);
    }
    if (!ok) *abort_v = 1;
    l_sh[hh][row] = l_run;
    if (ok && !__all_sync(0xffffffffu, mbar_wait(&bar_o[(nsub - 1) & 1], ((nsub - 1) >> 1) & 1, WAIT_LIMIT_NS))) {
      ok = false;
      *abort_v = 1;
      if ((tid & 31) == 0) report_timeout(a.status, 0x702);
    }
  }
  const bool failed = __syncthreads_or(!ok);   // also: l_sh complete
  if (mma_thread && failed) {   // copies issued and not consumed land before the buffers are reused
    for (int j = (k_issued > 2 ? k_issued - 2 : 0); j < k_issued; ++j) mbar_wait(&kfull[j & 1], (j >> 1) & 1, WAIT_LIMIT_NS);
    for (int j = (v_issued > 2 ? v_issued - 2 : 0); j < v_issued; ++j) mbar_wait(&vfull[j & 1], (j >> 1) & 1, WAIT_LIMIT_NS);
  }
  tc_fence_after();
  if (tid == 0) TL(3);

  const float l_tot = l_sh[0][row] + l_sh[1][row];
  const int rr = row0 + row;                         // this thread's row of the group
  const bool rv = sm_thread && row < Rv && !failed;
  const int jq = g * G + rr / a.H, iq = rr % a.H;    // query head, action row
  const float inv_sa = (a.fp8 && a.s_a) ? 1.0f / *a.s_a : 1.0f;
  // writes 16 consecutive output features d0.. of row (token t, head jq)
  auto store16 = [&](int t, int jh, int d0, const float* v) {
    const int kidx = jh * DH + d0;
    const size_t ob = a.o_rowmajor ? (static_cast<size_t>(t) * a.Hq * DH + kidx) * 2
                    : a.fp8 ? btile_offset(t, kidx, a.Nt, a.NKC_o) : btile_offset(t, 2 * kidx + 16, a.Nt, a.NKC_o);
    if (!in_bounds(a.status, ob + (a.o_rowmajor ? 31 : 15), a.o_extent, 0x9011)) return;
    if (a.o_rowmajor) {
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(t) * a.Hq * DH + kidx);
      dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
      dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                          pack_bf16x2(v[14], v[15]));
    } else if (a.fp8) {
      *reinterpret_cast<uint4*>(a.o + btile_offset(t, kidx, a.Nt, a.NKC_o)) =
          make_uint4(pack_e4m3x4(v[0] * inv_sa, v[1] * inv_sa, v[2] * inv_sa, v[3] * inv_sa),
                     pack_e4m3x4(v[4] * inv_sa, v[5] * inv_sa, v[6] * inv_sa, v[7] * inv_sa),
                     pack_e4m3x4(v[8] * inv_sa, v[9] * inv_sa, v[10] * inv_sa, v[11] * inv_sa),
                     pack_e4m3x4(v[12] * inv_sa, v[13] * inv_sa, v[14] * inv_sa, v[15] * inv_sa));
    } else {
      *reinterpret_cast<uint4*>(a.o + btile_offset(t, 2 * kidx, a.Nt, a.NKC_o)) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
      *reinterpret_cast<uint4*>(a.o + btile_offset(t, 2 * kidx + 16, a.Nt, a.NKC_o)) =
          make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                     pack_bf16x2(v[14], v[15]));
    }
  };

  if (sm_thread && C == 1) {   // the copy / MMA warp holds no rows
    const float inv = 1.0f / l_tot;
#pragma unroll 1
    for (int c0 = hh * (DH / 2); c0 < (hh + 1) * (DH / 2); c0 += 16) {   // this thread's half of the row
      uint32_t ov[16];
      tmem_ld16_nowait(tO + lane_base + c0, ov);
      tmem_wait_ld();
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(ov[e]) * inv;
      if (rv) store16(b * a.H + iq, jq, c0, v);
    }
  } else if (sm_thread) {
    // this chunk's (O, max, sum) row into the scratch, [B][Hq][C][H][OLD]
    float* xrow = a.xscratch + ((static_cast<size_t>(b) * a.Hq + jq) * C + c) * a.H * OLD + static_cast<size_t>(iq) * OLD;
#pragma unroll 1
    for (int c0 = hh * (DH / 2); c0 < (hh + 1) * (DH / 2); c0 += 16) {   // this thread's half of the row
      uint32_t ov[16];
      tmem_ld16_nowait(tO + lane_base + c0, ov);
      tmem_wait_ld();
      if (rv)
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(xrow + c0 + e) = make_float4(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1]),
                                                                  __uint_as_float(ov[e + 2]), __uint_as_float(ov[e + 3]));
    }
    if (rv && hh == 0) *reinterpret_cast<float4*>(xrow + DH) = make_float4(m_run, l_tot, 0.f, 0.f);
    // the peers fetch these rows with bulk copies (async proxy): order this thread's generic-proxy
    // stores before them, ahead of the cluster barrier's release
    fence_proxy_async_global();
  }
  tc_fence_before();
  fence_proxy_async_smem();   // the staging below overwrites Q/K/V/P by bulk copy
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, gm.tcols);
  }
  if (C == 1) {
    if (tid == 0) TL(5);
    return;
  }
  cluster_arrive_release();   // every chunk's rows are in the scratch after this barrier
  cluster_wait_acquire();
  if (tid == 0) TL(6);
  // ---------------- merge the rows this CTA owns over the key chunks, in rank order
  const int r_lo = c * Rv / C, r_hi = (c + 1) * Rv / C;
  const int RM = (128 + C - 1) / C;                  // staged rows per chunk (upper bound of r_hi - r_lo)
  float* stage = reinterpret_cast<float*>(dsm);      // [C][RM][OLD]
  if (tid == 0) {
    mbar_arrive_expect_tx(&stage_bar, static_cast<uint32_t>(r_hi - r_lo) * OLD * 4u * C);
    for (int r = r_lo; r < r_hi;) {                  // runs of rows within one query head
      const int gr = row0 + r, jh = g * G + gr / a.H, ih = gr % a.H;
      const int run = min(r_hi - r, a.H - ih);
      for (int s2 = 0; s2 < C; ++s2)
        bulk_g2s(stage + (static_cast<size_t>(s2) * RM + (r - r_lo)) * OLD,
                 a.xscratch + ((static_cast<size_t>(b) * a.Hq + jh) * C + s2) * a.H * OLD + static_cast<size_t>(ih) * OLD,
                 static_cast<uint32_t>(run) * OLD * 4u, &stage_bar);
      r += run;
    }
  }
  if (!mbar_wait(&stage_bar, 0, WAIT_LIMIT_NS) && tid == 0) report_timeout(a.status, 0x703);
  if (tid == 0) TL(4);
  float* w_sh = reinterpret_cast<float*>(dsm + gm.w_off);   // [16][128]: merge weight of chunk s2, owned row
  const int nr = r_hi - r_lo;
  if (tid < nr) {
    float mv[16], lv[16];
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2) {
      if (s2 < C) {
        const float2 ml = *reinterpret_cast<const float2*>(stage + (static_cast<size_t>(s2) * RM + tid) * OLD + DH);
        mv[s2] = ml.x;
        lv[s2] = ml.y;
      } else {
        mv[s2] = -INFINITY;
        lv[s2] = 0.f;
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2) M = fmaxf(M, mv[s2]);
    float den = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2) {
      if (s2 < C) {
        const float e = exp2f(mv[s2] - M);
        w_sh[s2 * 128 + tid] = e;
        den += e * lv[s2];
      }
    }
    inv_den[tid] = 1.0f / den;
  }
  __syncthreads();
  if (tid == 0) TL(7);
  // 16 output features per work item: (owned row, 16-feature group)
  for (int it = tid; it < nr * (DH / 16); it += UA_THREADS) {
    const int rq = it / (DH / 16), d0 = (it % (DH / 16)) * 16;
    const int gr = row0 + r_lo + rq, jh = g * G + gr / a.H, ih = gr % a.H;
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2)
      if (s2 < C) {
        const float w = w_sh[s2 * 128 + rq];
        const float* src = stage + (static_cast<size_t>(s2) * RM + rq) * OLD + d0;
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 v = *reinterpret_cast<const float4*>(src + e);
          acc[e] += w * v.x;   // rank order
          acc[e + 1] += w * v.y;
          acc[e + 2] += w * v.z;
          acc[e + 3] += w * v.w;
        }
      }
    const float id = inv_den[rq];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] *= id;
    store16(b * a.H + ih, jh, d0, acc);
  }
  __syncthreads();
  if (tid == 0) TL(5);
}

// ================================================================== in-proj and final

__global__ void __launch_bounds__(256) k_inproj_tc(const __grid_constant__ InprojArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ uint64_t wbar;
  __shared__ float xs[64];
  __shared__ float part[16][4];
  TL_DECL
  TL_BEGIN(1);
  __nv_bfloat16* wsm = reinterpret_cast<__nv_bfloat16*>(dsm);   // [A][D]: consecutive threads read consecutive n
  const int tid = threadIdx.x;
  const uint32_t wbytes = static_cast<uint32_t>(a.D) * a.A * 2;
  const bool emb = a.emb != nullptr;   // prefix pass: h is the embedded token itself
  if (tid == 0) {
    mbar_init(&wbar, 1);
    fence_mbar_init();
    if (!emb) {
      mbar_arrive_expect_tx(&wbar, wbytes);
      bulk_g2s(wsm, a.w_in, wbytes, &wbar);   // static weights: before the dependency wait
    }
  }
  grid_dep_launch();
  constexpr int QMAX = 16;                 // D <= 4096
  float base[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int n = tid + q * 256;
    base[q] = (n < a.D && !emb) ? a.b_in[n] + (a.temb ? a.temb[n] : 0.f) : 0.f;   // no temb: adaptive RMSNorm
  }
  grid_dep_wait();
  if (tid == 0) TL(1);
  if (!emb && !mbar_wait(&wbar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x800);
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {   // the weights are staged once per CTA
  if (!emb && tid < a.A) xs[tid] = __bfloat162float(__float2bfloat16_rn(a.x[static_cast<size_t>(t) * a.A + tid]));
  __syncthreads();
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int n = tid + q * 256;
    if (q * 256 >= a.D) continue;   // uniform across the block
    float hv = 0.f;
    if (n < a.D) {
      if (emb) {
        hv = __bfloat162float(a.emb[static_cast<size_t>(t) * a.D + n]);
      } else {
        float acc = 0.f;
        for (int i = 0; i < a.A; ++i) acc = fmaf(__bfloat162float(wsm[static_cast<size_t>(i) * a.D + n]), xs[i], acc);
        hv = acc + base[q];
      }
      a.h[htile_offset(t, n, a.Nt, a.KB)] = hv;
      if (a.xb)
        *reinterpret_cast<__nv_bfloat16*>(a.xb + btile_offset(t, 2 * n, a.Nt, a.NKC_x)) =
            __float2bfloat16_rn(hv * a.xb_gamma[n]);
    }
    float sq = hv * hv;
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) part[2 * q + (warp >> 2)][warp & 3] = sq;
  }
  __syncthreads();
  const int nmb = (a.D + BM - 1) / BM;
  if (tid < nmb) a.ssq[static_cast<size_t>(t) * a.ssq_ld + tid] = ((part[tid][0] + part[tid][1]) + part[tid][2]) + part[tid][3];
  __syncthreads();   // xs and part are rewritten by the next token
  }
  if (tid == 0) TL(5);
}

__global__ void __launch_bounds__(256) k_final_tc(const __grid_constant__ FinalArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ uint64_t wbar;
  __shared__ float ssq_sh[16];
  TL_DECL
  TL_BEGIN(2);
  __nv_bfloat16* wsm = reinterpret_cast<__nv_bfloat16*>(dsm);                     // [A][D]
  float* hn = reinterpret_cast<float*>(dsm + ((static_cast<size_t>(a.A) * a.D * 2 + 127) & ~size_t(127)));
  const int tid = threadIdx.x;
  const uint32_t wbytes = static_cast<uint32_t>(a.A) * a.D * 2;
  if (tid == 0) {
    mbar_init(&wbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&wbar, wbytes);
    bulk_g2s(wsm, a.w_out, wbytes, &wbar);   // static weights: before the dependency wait
  }
  grid_dep_launch();
  constexpr int QMAX = 16;
  float gf[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int k = tid + q * 256;
    gf[q] = k < a.D ? a.g_f[k] : 0.f;
  }
  grid_dep_wait();
  if (threadIdx.x == 0) TL(1);
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {   // the weights are staged once per CTA
  float hv[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int k = tid + q * 256;
    hv[q] = k < a.D ? a.h[htile_offset(t, k, a.Nt, a.KB)] : 0.f;
  }
  if (tid < a.ssq_parts) ssq_sh[tid] = a.ssq[static_cast<size_t>(t) * a.ssq_ld + tid];
  __syncthreads();
  float ss = 0.f;
  for (int p = 0; p < a.ssq_parts; ++p) ss += ssq_sh[p];
  const float r = 1.0f / sqrtf(ss / a.D + a.eps);
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int k = tid + q * 256;
    if (k < a.D) hn[k] = __bfloat162float(__float2bfloat16_rn(hv[q] * r * gf[q]));
  }
  __syncthreads();
  if (!mbar_wait(&wbar, 0, WAIT_LIMIT_NS)) report_timeout(a.status, 0x801);
  const int warp = tid >> 5, lane = tid & 31;
  for (int i = warp; i < a.A; i += 8) {
    const __nv_bfloat16* wr = wsm + static_cast<size_t>(i) * a.D;
    float acc = 0.f;
    for (int k = lane; k < a.D; k += 32) acc = fmaf(__bfloat162float(wr[k]), hn[k], acc);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const size_t xi = static_cast<size_t>(t) * a.A + i;
      a.x_out[xi] = a.x_in[xi] + a.dt * (acc + a.b_out[i]);
    }
  }
  __syncthreads();   // hn and ssq_sh are rewritten by the next token
  }
  if (tid == 0) TL(5);
}

// [rows][cols] float32 -> [cols][rows] bf16
__global__ void k_to_bf16_t(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int rows, int cols) {
  const size_t n = static_cast<size_t>(rows) * cols;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t c = i / rows, r = i % rows;   // dst index i = c * rows + r
    dst[i] = __float2bfloat16_rn(src[r * cols + c]);
  }
}

__global__ void k_to_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// ================================================================== launch helpers

cudaError_t launch_ex(const void* func, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, int cluster_x,
                      void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  int n = 0;
  if (pdl) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster_x;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelExC(&cfg, func, args);
}

// Failure-detection self-test: one device wait on a barrier that nothing completes.  It gives
// up after limit_ns, latches the timeout bit with where-code 0x7F0, and the kernel returns.
__global__ void k_wait_selftest(unsigned* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns)) report_timeout(status, 0x7F0);
}

}  // namespace

size_t pt_smem_bytes(int Nt, int stages) { return pt_ring_bytes(Nt, stages) + PT_RED_TOK * RED_LD * 4; }

size_t gemm_smem_bytes(int Nt, int stages, int b_kind, int fp8, int S, int nk, int w4, int epi, int H, int xb,
                       int red_tok, int kpu) {
  return gemm_rope_off(Nt, stages, b_kind, fp8, S, nk, w4, epi, red_tok, kpu) + gemm_stage_bytes(epi, fp8, Nt, S, H, xb);
}

size_t gemm_scratch_bytes(int NT, int MB, int S, int Nt) {
  return S > 1 ? static_cast<size_t>(NT) * MB * S * Nt * BM * 4 : 0;
}

size_t attn_scratch_bytes(int B, int Hq, int C, int H, int dh) {
  return C > 1 ? static_cast<size_t>(B) * Hq * C * H * (dh + 4) * 4 : 0;
}

size_t attn_smem_bytes(int H, int dh, int KC, int C, int umma) {
  if (umma) return uattn_geom(dh).total;   // the merge stage (<= 144 rows x (dh + 4) floats) overlays it
  const AttnGeom g = attn_geom(H, dh, KC, C);
  const size_t compute = static_cast<size_t>(g.q_bytes) + g.kv_bytes;
  // the partial rows are staged over Q/K/V (obuf) before the merge stage overlays them
  const size_t merge = std::max<size_t>(g.obuf_bytes, C > 1 ? static_cast<size_t>(C) * g.R * g.rowb : 0);
  return compute > merge ? compute : merge;
}

const void* gemm_kernel(int epi, int fp8, int norm, int w4);

cudaError_t tc_kernels_init() {
  cudaError_t e;
  int dev = 0, optin = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const void* fns[] = {gemm_kernel(EPI_QKV, 0, 0, 0), gemm_kernel(EPI_RESID, 0, 0, 0), gemm_kernel(EPI_GELU, 0, 0, 0),
                       gemm_kernel(EPI_QKV, 1, 1, 0), gemm_kernel(EPI_GELU, 1, 1, 0), gemm_kernel(EPI_RESID, 1, 0, 0),
                       gemm_kernel(EPI_QKV, 0, 0, 1), gemm_kernel(EPI_RESID, 0, 0, 1), gemm_kernel(EPI_GELU, 0, 0, 1),
                       reinterpret_cast<const void*>(k_attn_tc<64>),
                       reinterpret_cast<const void*>(k_attn_tc<128>), reinterpret_cast<const void*>(k_attn_tc<256>),
                       reinterpret_cast<const void*>(k_attn_umma<64>),
                       reinterpret_cast<const void*>(k_attn_umma<128>), reinterpret_cast<const void*>(k_attn_umma<256>),
                       reinterpret_cast<const void*>(k_inproj_tc), reinterpret_cast<const void*>(k_final_tc),
                       reinterpret_cast<const void*>(k_gemm_gelu_pt)};
  for (const void* f : fns) {
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, f)) != cudaSuccess) return e;
    const int dyn = optin - static_cast<int>(fa.sharedSizeBytes);
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared)) !=
        cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Dynamic shared memory a GEMM CTA may use alone on an SM; 0 when the device cannot be queried (the
// plans then find that nothing fits and the launch reports it).
int max_dynamic_smem() {
  int dev = 0, optin = 0;
  cudaFuncAttributes fa{};
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, gemm_kernel(EPI_RESID, 0, 0, 0)) != cudaSuccess)
    return 0;
  return std::max(0, optin - static_cast<int>(fa.sharedSizeBytes));
}

// ... and when two GEMM CTAs share an SM (0 as above).
int pair_dynamic_smem() {
  int dev = 0, per_sm = 0, reserved = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return 0;
  int stat = 0;
  for (int epi : {EPI_QKV, EPI_RESID, EPI_GELU}) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, gemm_kernel(epi, 0, 0, 0)) != cudaSuccess) return 0;
    stat = std::max(stat, static_cast<int>(fa.sharedSizeBytes));
  }
  return std::max(0, per_sm / 2 - reserved - stat);
}

// One instantiation per (epilogue, operand type, B-operand kind, 4-bit weights) in use.
const void* gemm_kernel(int epi, int fp8, int norm, int w4) {
  if (w4) {
    if (fp8 || norm) return nullptr;
    if (epi == EPI_QKV) return reinterpret_cast<const void*>(k_gemm_tc<EPI_QKV, 0, 0, 1>);
    if (epi == EPI_RESID) return reinterpret_cast<const void*>(k_gemm_tc<EPI_RESID, 0, 0, 1>);
    if (epi == EPI_GELU) return reinterpret_cast<const void*>(k_gemm_tc<EPI_GELU, 0, 0, 1>);
  } else if (!fp8 && !norm) {
    if (epi == EPI_QKV) return reinterpret_cast<const void*>(k_gemm_tc<EPI_QKV, 0, 0, 0>);
    if (epi == EPI_RESID) return reinterpret_cast<const void*>(k_gemm_tc<EPI_RESID, 0, 0, 0>);
    if (epi == EPI_GELU) return reinterpret_cast<const void*>(k_gemm_tc<EPI_GELU, 0, 0, 0>);
  } else if (fp8 && norm) {
    if (epi == EPI_QKV) return reinterpret_cast<const void*>(k_gemm_tc<EPI_QKV, 1, 1, 0>);
    if (epi == EPI_GELU) return reinterpret_cast<const void*>(k_gemm_tc<EPI_GELU, 1, 1, 0>);
  } else if (fp8 && !norm) {
    if (epi == EPI_RESID) return reinterpret_cast<const void*>(k_gemm_tc<EPI_RESID, 1, 0, 0>);
  }
  return nullptr;
}

cudaError_t launch_gemm_tc(const GemmArgs& a, int n_tiles, cudaStream_t s, bool pdl) {
  GemmArgs copy = a;
  void* args[] = {&copy};
  if (a.persist) {
    if (a.epi != EPI_GELU || a.fp8 || a.w4 || a.b_kind != B_ROWS || a.S != 1 || a.pt_ctas < 1 ||
        a.pt_ctas > a.MB * n_tiles || a.Nt > 256 || a.NKC % PT_KPS != 0)
      return cudaErrorInvalidValue;
    copy.pt_nt = n_tiles;
    return launch_ex(reinterpret_cast<const void*>(k_gemm_gelu_pt), dim3(a.pt_ctas), dim3(PT_THREADS),
                     pt_smem_bytes(a.Nt, a.stages), s, pdl, 1, args);
  }
  const int nk_max = (a.NKC + a.S - 1) / a.S;
  const void* f = gemm_kernel(a.epi, a.fp8, a.b_kind == B_NORM, a.w4);
  if (!f) return cudaErrorInvalidValue;
  return launch_ex(f, dim3(a.S, n_tiles, a.MB), dim3(GEMM_THREADS),
                   gemm_smem_bytes(a.Nt, a.stages, a.b_kind, a.fp8, a.S, nk_max, a.w4, a.epi, a.H, a.xb_out != nullptr, a.red_tok,
                                   a.kpu), s,
                   pdl, a.S, args);
}

namespace {

// cuTensorMapEncodeTiled from the driver, found once through the runtime (no link-time dependency).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map of K or V ([planes][keys][dh] bf16, planes plane_bytes apart), 128-byte swizzle; keys past
// `keys` read as zeros.  one_box: the 4-D view (64 features, keys, dh/64 feature blocks, planes) with
// boxes of 64 x 64 x dh/64 x 1, which land as [feature block][key][128 B] in one copy; otherwise the
// 3-D view (dh, keys, planes) with boxes of 64 features x 64 keys.
bool encode_kv_map(CUtensorMap* m, const void* base, uint64_t dh, uint64_t keys, uint64_t planes,
                   uint64_t plane_bytes, bool one_box) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn || !base || (reinterpret_cast<uintptr_t>(base) & 15u) || keys == 0 || planes == 0 || dh % 64 != 0)
    return false;
  const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  if (one_box) {
    const cuuint64_t dims[4] = {64, keys, dh / 64, planes};
    const cuuint64_t strides[3] = {dh * 2, 128, plane_bytes};
    const cuuint32_t box[4] = {64u, 64u, static_cast<cuuint32_t>(dh / 64), 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4u, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  const cuuint64_t dims[3] = {dh, keys, planes};
  const cuuint64_t strides[2] = {dh * 2, plane_bytes};
  const cuuint32_t box[3] = {64u, 64u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3u, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention_tc(const AttnArgs& a, int B, cudaStream_t s, bool pdl) {
  AttnArgs copy = a;
  void* args[] = {&copy};
  const size_t smem = attn_smem_bytes(a.H, a.dh, a.KC, a.C, a.umma);
  if (a.umma) {
    // K and V [B][Hkv][S_max][dh] as B*Hkv planes of this call's P + H keys (keys past them read as zeros)
    const uint64_t dh = static_cast<uint64_t>(a.dh), keys = static_cast<uint64_t>(a.P + a.H);
    const uint64_t planes = static_cast<uint64_t>(B) * a.Hkv, pb = static_cast<uint64_t>(a.S_max) * dh * 2;
    // one copy per sub-chunk where the driver accepts the 4-D view, else dh/64 copies
    copy.kv_boxes = 1;
    if (!encode_kv_map(&copy.tm_k, a.kv_k, dh, keys, planes, pb, true) ||
        !encode_kv_map(&copy.tm_v, a.kv_v, dh, keys, planes, pb, true)) {
      copy.kv_boxes = static_cast<int>(dh / 64);
      if (!encode_kv_map(&copy.tm_k, a.kv_k, dh, keys, planes, pb, false) ||
          !encode_kv_map(&copy.tm_v, a.kv_v, dh, keys, planes, pb, false))
        return cudaErrorInvalidValue;
    }
    const void* f = a.dh == 64 ? reinterpret_cast<const void*>(k_attn_umma<64>)
                  : a.dh == 128 ? reinterpret_cast<const void*>(k_attn_umma<128>)
                                : reinterpret_cast<const void*>(k_attn_umma<256>);
    const int tiles = (a.Hq / a.Hkv * a.H + 127) / 128;
    return launch_ex(f, dim3(a.C, a.Hkv * tiles, B), dim3(UA_THREADS), smem, s, pdl, a.C, args);
  }
  const int Hp = (a.H + 15) & ~15;
  const int nw = min(8, max(4, Hp / 16));
  const void* f = a.dh == 64 ? reinterpret_cast<const void*>(k_attn_tc<64>)
                : a.dh == 128 ? reinterpret_cast<const void*>(k_attn_tc<128>)
                              : reinterpret_cast<const void*>(k_attn_tc<256>);
  return launch_ex(f, dim3(a.C, a.Hq, B), dim3(32 * nw), smem, s, pdl, a.C, args);
}

cudaError_t launch_inproj_tc(const InprojArgs& a, cudaStream_t s, bool pdl) {
  InprojArgs copy = a;
  void* args[] = {&copy};
  return launch_ex(reinterpret_cast<const void*>(k_inproj_tc), dim3(a.max_ctas > 0 && a.max_ctas < a.T ? a.max_ctas : a.T), dim3(256),
                   static_cast<size_t>(a.D) * a.A * 2, s, pdl, 1, args);
}

cudaError_t launch_final_tc(const FinalArgs& a, cudaStream_t s, bool pdl) {
  FinalArgs copy = a;
  void* args[] = {&copy};
  const size_t smem = ((static_cast<size_t>(a.A) * a.D * 2 + 127) & ~size_t(127)) + static_cast<size_t>(a.D) * 4;
  return launch_ex(reinterpret_cast<const void*>(k_final_tc), dim3(a.max_ctas > 0 && a.max_ctas < a.T ? a.max_ctas : a.T),
                   dim3(256), smem, s, pdl, 1, args);
}

cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s) {
  k_to_bf16<<<static_cast<unsigned>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024), 256, 0, s>>>(src, dst, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(unsigned* status, unsigned long long limit_ns, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_to_bf16_t(const float* src, __nv_bfloat16* dst, int rows, int cols, cudaStream_t s) {
  const size_t n = static_cast<size_t>(rows) * cols;
  k_to_bf16_t<<<static_cast<unsigned>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024), 256, 0, s>>>(src, dst, rows, cols);
  return cudaGetLastError();
}

const void* inproj_kernel_ptr() { return reinterpret_cast<const void*>(k_inproj_tc); }
const void* final_kernel_ptr() { return reinterpret_cast<const void*>(k_final_tc); }

}  // namespace tc
}  // namespace fr

#ifdef FR_TIMELINE
extern "C" int fr_debug_timeline(unsigned long long* dev_buf, unsigned cap, unsigned* count_out) {
  unsigned zero = 0;
  if (count_out) {
    cudaDeviceSynchronize();
    cudaMemcpyFromSymbol(count_out, fr::tc::g_tl_count, sizeof(unsigned));
  }
  cudaMemcpyToSymbol(fr::tc::g_tl, &dev_buf, sizeof(dev_buf));
  cudaMemcpyToSymbol(fr::tc::g_tl_cap, &cap, sizeof(cap));
  cudaMemcpyToSymbol(fr::tc::g_tl_count, &zero, sizeof(zero));
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : -4;
}
#endif
