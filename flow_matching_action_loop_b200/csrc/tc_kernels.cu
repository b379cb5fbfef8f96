// Tensor-core kernels of the action-expert loop (sm_100a).
//
// GEMM (swap-AB): D[128 features x Nt tokens] = W_tile[128 x K] * act[Nt x K]^T
//   on tcgen05 with the accumulator in tensor memory.  Weights are the A operand,
//   pre-tiled by the packer so that each pipeline chunk (128 rows x 128 bytes of K)
//   is one contiguous 16 KB block moved by a single bulk copy.  The B operand
//   (activations) is staged by warps 2-7: RMSNorm (+ bf16/e4m3 quantisation) is
//   fused into this staging for the QKV and gate|up projections (FlashRT
//   walkthrough, component 8: norm and residual+norm+quant fusion).  Split-K is a
//   thread-block cluster: partial tiles are summed over distributed shared memory
//   in rank order, then a fused epilogue runs:
//     EPI_QKV   QKV split + rotate-half RoPE, q to its buffer, k/v into the KV cache
//     EPI_RESID residual add into h and the per-token sum of squares of the new h
//     EPI_GELU  GeLU(tanh)(gate) * up, quantised for the down projection
//   (PhyAI page, optimisation paragraph: fused QKV and merged gate|up GEMMs.)
//
// Attention: one cluster per (sample, query head), one CTA per key chunk.  Warp-level
//   bf16 MMA computes scores and P*V with an online softmax over 64-key sub-chunks;
//   the key chunks are merged with their log-sum-exp weights over distributed shared
//   memory in rank order (flash-decoding split over keys).
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"
#include "sm100.h"
#include "tc_kernels.h"

namespace cg = cooperative_groups;

namespace fr {
namespace tc {
namespace {

using namespace fr::sm100;

constexpr int RED_LD = BM + 4;   // row stride (floats) of the epilogue reduction buffer

__device__ __forceinline__ void report_timeout(unsigned* status, uint32_t where) {
  if (status) {
    atomicOr(status, ST_TIMEOUT_BIT);
    atomicExch(status + 1, where);
    atomicExch(status + 2, blockIdx.x | (blockIdx.y << 8) | (blockIdx.z << 20));
  }
}

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float gelu_tanh(float g) {
  const float c0 = 0.7978845608028654f;   // sqrt(2/pi)
  return 0.5f * g * (1.f + tanhf(c0 * (g + 0.044715f * g * g * g)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ================================================================== GEMM

struct GemmSmem {
  uint64_t full_a[MAX_STAGES];
  uint64_t full_b[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  float rstd[NT_MAX];
  float ssq_part[2][4];
};

__global__ void __launch_bounds__(GEMM_THREADS, 2) k_gemm_tc(const __grid_constant__ GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t dsm[];
  __shared__ GemmSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ks = blockIdx.x;            // split-K rank (cluster rank)
  const int mb = blockIdx.y;            // m-block
  const int nt = blockIdx.z;            // n-tile
  const int Nt = a.Nt;
  const int n0 = nt * Nt;               // first token of this tile
  const int kc0 = ks * a.NKC / a.S, kc1 = (ks + 1) * a.NKC / a.S;
  const int nk = kc1 - kc0;
  const int stages = a.stages;
  const uint32_t A_BYTES = BM * KCB;
  const uint32_t B_BYTES = static_cast<uint32_t>(Nt) * KCB;
  const uint32_t SLOT = A_BYTES + B_BYTES;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&sh.full_a[s], 1);
      mbar_init(&sh.full_b[s], 192);
      mbar_init(&sh.empty[s], 1);
    }
    mbar_init(&sh.done, 1);
    sh.abort_flag = 0;
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
  grid_dep_launch();   // the next kernel may start its own weight prefetch now
  const uint32_t tacc = sh.tmem_base;

  if (warp == 0) {
    // ---------------- A producer: weight chunks by bulk copy (independent of the previous kernel)
    if (lane == 0) {
      const uint8_t* wsrc = a.W + (static_cast<size_t>(mb) * a.NKC + kc0) * A_BYTES;
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        if (i >= stages && !mbar_wait(&sh.empty[s], ((i / stages) - 1) & 1, WAIT_LIMIT_NS)) {
          report_timeout(a.status, 0x100);
          sh.abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&sh.full_a[s], A_BYTES);
        bulk_g2s(dsm + s * SLOT, wsrc + static_cast<size_t>(i) * A_BYTES, A_BYTES, &sh.full_a[s]);
        issued = i + 1;
      }
      // drain: every copy issued into this CTA's shared memory has landed before it is reused
      for (int i = (issued > stages ? issued - stages : 0); i < issued; ++i)
        mbar_wait(&sh.full_a[i % stages], (i / stages) & 1, WAIT_LIMIT_NS);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(a.fp8 ? FMT_E4M3 : FMT_BF16, BM, Nt);
      for (int i = 0; i < nk; ++i) {
        const int s = i % stages;
        const uint32_t par = (i / stages) & 1;
        if (!mbar_wait(&sh.full_a[s], par, WAIT_LIMIT_NS) || !mbar_wait(&sh.full_b[s], par, WAIT_LIMIT_NS)) {
          report_timeout(a.status, 0x200);
          sh.abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(dsm + s * SLOT), b0 = a0 + A_BYTES;
#pragma unroll
        for (int k = 0; k < KCB / 32; ++k) {
          const uint64_t ad = smem_desc(a0 + k * 2 * BM * 16, BM * 16, 128);
          const uint64_t bd = smem_desc(b0 + k * 2 * Nt * 16, Nt * 16, 128);
          if (a.fp8) mma_e4m3(tacc, ad, bd, idesc, (i | k) != 0);
          else mma_bf16(tacc, ad, bd, idesc, (i | k) != 0);
        }
        mma_commit(&sh.empty[s]);
      }
      mma_commit(&sh.done);
    }
  } else {
    // ---------------- B staging (warps 2-7): activations of this n-tile into the ring
    grid_dep_wait();
    const int st = tid - 64;   // 0..191
    if (a.b_kind == B_NORM) {
      for (int r = st; r < Nt; r += 192) {
        const int t = n0 + r;
        float ss = 0.f;
        if (t < a.T)
          for (int p = 0; p < a.ssq_parts; ++p) ss += a.ssq[p * a.T_pad + t];
        sh.rstd[r] = 1.0f / sqrtf(ss / a.Kdim + a.eps);
      }
      asm volatile("bar.sync 1, 192;" ::: "memory");
    }
    const float inv_sa = (a.fp8 && a.b_kind == B_NORM) ? 1.0f / *a.s_a : 1.0f;
    const int elem = a.fp8 ? 1 : 2;
    const int kel = KCB / elem;                 // K elements per chunk
    for (int i = 0; i < nk; ++i) {
      const int s = i % stages;
      if (i >= stages && !mbar_wait(&sh.empty[s], ((i / stages) - 1) & 1, WAIT_LIMIT_NS)) {
        report_timeout(a.status, 0x300);
        sh.abort_flag = 1;
        break;
      }
      uint8_t* bdst = dsm + s * SLOT + A_BYTES;
      const int k0 = (kc0 + i) * kel;
      // item = one 16-byte row segment (slab j of token row r)
      for (int it = st; it < Nt * 8; it += 192) {
        const int r = it >> 3, j = it & 7;
        const int t = n0 + r;
        const int kk = k0 + j * (16 / elem);
        uint4 val = make_uint4(0, 0, 0, 0);
        if (t < a.T && kk < a.Kdim) {
          if (a.b_kind == B_ROWS) {
            val = *reinterpret_cast<const uint4*>(a.act + (static_cast<size_t>(t) * a.act_ld + kk) * elem);
          } else {
            const float* hp = a.h + static_cast<size_t>(t) * a.Kdim + kk;
            const float* gp = a.gamma + kk;
            const float rs = sh.rstd[r];
            if (!a.fp8) {
              const float4 h0 = *reinterpret_cast<const float4*>(hp), h1 = *reinterpret_cast<const float4*>(hp + 4);
              const float4 g0 = *reinterpret_cast<const float4*>(gp), g1 = *reinterpret_cast<const float4*>(gp + 4);
              val.x = pack_bf16x2(h0.x * rs * g0.x, h0.y * rs * g0.y);
              val.y = pack_bf16x2(h0.z * rs * g0.z, h0.w * rs * g0.w);
              val.z = pack_bf16x2(h1.x * rs * g1.x, h1.y * rs * g1.y);
              val.w = pack_bf16x2(h1.z * rs * g1.z, h1.w * rs * g1.w);
            } else {
              uint32_t wds[4];
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const float4 hv = *reinterpret_cast<const float4*>(hp + 4 * q4);
                const float4 gv = *reinterpret_cast<const float4*>(gp + 4 * q4);
                wds[q4] = static_cast<uint32_t>(to_e4m3(hv.x * rs * gv.x * inv_sa)) |
                          (static_cast<uint32_t>(to_e4m3(hv.y * rs * gv.y * inv_sa)) << 8) |
                          (static_cast<uint32_t>(to_e4m3(hv.z * rs * gv.z * inv_sa)) << 16) |
                          (static_cast<uint32_t>(to_e4m3(hv.w * rs * gv.w * inv_sa)) << 24);
              }
              val = make_uint4(wds[0], wds[1], wds[2], wds[3]);
            }
          }
        }
        *reinterpret_cast<uint4*>(bdst + j * Nt * 16 + (r >> 3) * 128 + (r & 7) * 16) = val;
      }
      fence_proxy_async_smem();   // generic-proxy writes -> visible to the tensor core (async proxy)
      mbar_arrive(&sh.full_b[s]);
    }
  }

  // ---------------- epilogue
  grid_dep_wait();
  if (!mbar_wait(&sh.done, 0, WAIT_LIMIT_NS)) {
    report_timeout(a.status, 0x400);
    sh.abort_flag = 1;
  }
  tc_fence_after();
  __syncthreads();
  float* red = reinterpret_cast<float*>(dsm);          // [Nt][RED_LD], aliases the drained ring
  if (warp >= 4) {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    for (int c0 = 0; c0 < Nt; c0 += 16) {
      float v[16];
      tmem_ld16(tacc + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) red[(c0 + j) * RED_LD + row] = v[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  cg::cluster_group cluster = cg::this_cluster();
  if (a.S > 1) cluster.sync();

  const float al = a.alpha ? *a.alpha : 1.0f;
  const int tok0 = ks * Nt / a.S, tok1 = (ks + 1) * Nt / a.S;
  // split-K sum of one accumulator element over the cluster, in rank order (deterministic)
  auto gather = [&](int tok, int row) -> float {
    const int idx = tok * RED_LD + row;
    if (a.S == 1) return red[idx] * al;
    float v = 0.f;
    for (int s = 0; s < a.S; ++s) v += cluster.map_shared_rank(red, s)[idx];
    return v * al;
  };

  if (a.epi == EPI_RESID) {
    const int row = tid & 127, sub = tid >> 7;
    const int f = mb * BM + row;
    for (int tb = tok0; tb < tok1; tb += 2) {
      const int tok = tb + sub;
      const int t = n0 + tok;
      float sq = 0.f;
      if (tok < tok1 && t < a.T && f < a.Nout) {
        float* hp = a.h_out + static_cast<size_t>(t) * a.D + f;
        const float hv = *hp + gather(tok, row);
        *hp = hv;
        sq = hv * hv;
      }
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (lane == 0) sh.ssq_part[sub][(tid >> 5) & 3] = sq;
      __syncthreads();
      if (row == 0 && tok < tok1 && t < a.T_pad)
        a.ssq_out[mb * a.T_pad + t] = ((sh.ssq_part[sub][0] + sh.ssq_part[sub][1]) + sh.ssq_part[sub][2]) +
                                      sh.ssq_part[sub][3];
      __syncthreads();
    }
  } else if (a.epi == EPI_GELU) {
    const int p = tid & 63, sub = tid >> 6;
    const int f = mb * 64 + p;
    const float inv = (a.fp8 && a.s_a_out) ? 1.0f / *a.s_a_out : 1.0f;
    for (int tok = tok0 + sub; tok < tok1; tok += 4) {
      const int t = n0 + tok;
      if (t >= a.T || f >= a.F) continue;
      const float u = gelu_tanh(gather(tok, p)) * gather(tok, p + 64);
      if (a.fp8) a.u_out[static_cast<size_t>(t) * a.F + f] = to_e4m3(u * inv);
      else reinterpret_cast<__nv_bfloat16*>(a.u_out)[static_cast<size_t>(t) * a.F + f] = __float2bfloat16_rn(u);
    }
  } else {   // EPI_QKV
    const int half = a.dh >> 1;
    if (mb < a.MB_rot) {
      const int p = tid & 63, sub = tid >> 6;
      const int pi = mb * 64 + p;
      const int head = pi / half, j = pi % half;
      for (int tok = tok0 + sub; tok < tok1; tok += 4) {
        const int t = n0 + tok;
        if (t >= a.T) continue;
        const int b = t / a.H, i = t % a.H, pos = a.P + i;
        const float lo = gather(tok, p), hi = gather(tok, p + 64);
        const float c = a.rope_cos[pos * half + j], sn = a.rope_sin[pos * half + j];
        const float r0 = lo * c - hi * sn, r1 = lo * sn + hi * c;
        __nv_bfloat16* dst;
        if (head < a.Hq) dst = a.q_out + ((static_cast<size_t>(b) * a.Hq + head) * a.H + i) * a.dh;
        else dst = a.kv_k + ((static_cast<size_t>(b) * a.Hkv + (head - a.Hq)) * a.S_max + pos) * a.dh;
        dst[j] = __float2bfloat16_rn(r0);
        dst[j + half] = __float2bfloat16_rn(r1);
      }
    } else {
      const int row = tid & 127, sub = tid >> 7;
      const int idx = (mb - a.MB_rot) * BM + row;
      const int g = idx / a.dh, d = idx % a.dh;
      for (int tok = tok0 + sub; tok < tok1; tok += 2) {
        const int t = n0 + tok;
        if (t >= a.T) continue;
        const int b = t / a.H, i = t % a.H, pos = a.P + i;
        a.kv_v[((static_cast<size_t>(b) * a.Hkv + g) * a.S_max + pos) * a.dh + d] = __float2bfloat16_rn(gather(tok, row));
      }
    }
  }
  if (a.S > 1) cluster.sync();   // peers have finished reading this CTA's partial tile
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tacc, ncols);
  }
}

// ================================================================== attention

constexpr int SUBK = 64;          // keys per online-softmax step (the key chunk is a multiple of it)
constexpr int ATT_PAD = 8;        // bf16 elements of row padding (16 bytes) against bank conflicts

__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sdst)), "l"(gsrc), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int DH>
__global__ void __launch_bounds__(256) k_attn_tc(const __grid_constant__ AttnArgs a) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ float m_sh[256], l_sh[256];
  __shared__ float w_sh[16][32];
  constexpr int LD = DH + ATT_PAD;       // bf16 row stride in shared memory
  const int c = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
  const int g = (j * a.Hkv) / a.Hq;      // consecutive query-head groups share a KV head
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const int H = a.H, Hp = (H + 15) & ~15;
  const int S = a.P + H;
  const int key0 = c * a.KC;
  const int nkeys = min(a.KC, S - key0);
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(dsm);
  __nv_bfloat16* Ks = Qs + Hp * LD;
  __nv_bfloat16* Vs = Ks + a.KC * LD;
  const __nv_bfloat16* kg = a.kv_k + ((static_cast<size_t>(b) * a.Hkv + g) * a.S_max) * DH;
  const __nv_bfloat16* vg = a.kv_v + ((static_cast<size_t>(b) * a.Hkv + g) * a.S_max) * DH;
  constexpr int VPR = DH / 8;            // 16-byte vectors per row
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

  const int gq = lane >> 2, tq = lane & 3;
  const float sl2 = a.scale * 1.4426950408889634f;   // scores in log2 units
  float* Obuf = reinterpret_cast<float*>(Ks);         // [Hp][DH] fp32, reused after the keys are consumed
  const int n_rg = Hp / 16;
  // each warp owns row groups rg = warp, warp + nw, ...
  float oacc[DH / 8][4];
  float mrow[2], lrow[2];
  for (int rg0 = 0; rg0 < n_rg; rg0 += nw) {
    const int rg = rg0 + warp;
    const bool active = rg < n_rg;
    if (active) {
#pragma unroll
      for (int n = 0; n < DH / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
      mrow[0] = mrow[1] = -INFINITY;
      lrow[0] = lrow[1] = 0.f;
      const uint32_t qa = smem_u32(Qs + (rg * 16 + (lane & 15)) * LD + (lane >> 4) * 8);
      for (int kb = 0; kb < nkeys; kb += SUBK) {
        float sacc[SUBK / 8][4];
#pragma unroll
        for (int n = 0; n < SUBK / 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(qa + kk * 32, a0, a1, a2, a3);
#pragma unroll
          for (int n = 0; n < SUBK / 8; ++n) {
            uint32_t b0, b1;
            const uint32_t ka = smem_u32(Ks + (kb + n * 8 + (lane & 7)) * LD + kk * 16 + ((lane >> 3) & 1) * 8);
            ldsm_x2(ka, b0, b1);
            mma16816(sacc[n], a0, a1, a2, a3, b0, b1);
          }
        }
        // scale, mask, online softmax
        float mnew[2] = {mrow[0], mrow[1]};
#pragma unroll
        for (int n = 0; n < SUBK / 8; ++n) {
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
        for (int n = 0; n < SUBK / 8; ++n) {
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
        // O += P V
#pragma unroll
        for (int kk = 0; kk < SUBK / 16; ++kk) {
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
    __syncthreads();   // all warps are done with Ks/Vs of this pass before Obuf overwrites them
    if (active) {
      const int r0 = rg * 16 + gq;
#pragma unroll
      for (int n = 0; n < DH / 8; ++n) {
        const int col = n * 8 + tq * 2;
        Obuf[r0 * DH + col] = oacc[n][0];
        Obuf[r0 * DH + col + 1] = oacc[n][1];
        Obuf[(r0 + 8) * DH + col] = oacc[n][2];
        Obuf[(r0 + 8) * DH + col + 1] = oacc[n][3];
      }
      if (tq == 0) {
        m_sh[r0] = mrow[0];
        l_sh[r0] = lrow[0];
        m_sh[r0 + 8] = mrow[1];
        l_sh[r0 + 8] = lrow[1];
      }
    }
  }
  __syncthreads();
  // ---------------- merge the key chunks of this (sample, head) over the cluster, in rank order
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  const int C = a.C;
  const int r_lo = c * H / C, r_hi = (c + 1) * H / C;   // this CTA writes rows [r_lo, r_hi)
  const float inv_sa = (a.fp8 && a.s_a) ? 1.0f / *a.s_a : 1.0f;
  for (int rb = r_lo; rb < r_hi; rb += 16) {
    const int nr = min(16, r_hi - rb);
    // weights of each chunk for these rows: w_s = 2^(m_s - M) / sum_s 2^(m_s - M) l_s
    if (tid < nr) {
      const int r = rb + tid;
      float M = -INFINITY;
      for (int s = 0; s < C; ++s) M = fmaxf(M, cluster.map_shared_rank(m_sh, s)[r]);
      float den = 0.f;
      for (int s = 0; s < C; ++s) {
        const float e = exp2f(cluster.map_shared_rank(m_sh, s)[r] - M);
        w_sh[s][tid] = e;
        den += e * cluster.map_shared_rank(l_sh, s)[r];
      }
      const float inv = 1.0f / den;
      for (int s = 0; s < C; ++s) w_sh[s][tid] *= inv;
    }
    __syncthreads();
    for (int it = tid; it < nr * DH; it += blockDim.x) {
      const int rr = it / DH, d = it % DH;
      const int r = rb + rr;
      float acc = 0.f;
      for (int s = 0; s < C; ++s) acc += w_sh[s][rr] * cluster.map_shared_rank(Obuf, s)[r * DH + d];
      const size_t oi = (static_cast<size_t>(b) * H + r) * (a.Hq * DH) + static_cast<size_t>(j) * DH + d;
      if (a.fp8) a.o[oi] = to_e4m3(acc * inv_sa);
      else reinterpret_cast<__nv_bfloat16*>(a.o)[oi] = __float2bfloat16_rn(acc);
    }
    __syncthreads();
  }
  cluster.sync();   // peers have finished reading this CTA's partials
}

// ================================================================== in-proj and final

__global__ void __launch_bounds__(128) k_inproj_tc(const __grid_constant__ InprojArgs a) {
  extern __shared__ float xs[];
  __shared__ float wpart[4];
  grid_dep_launch();
  grid_dep_wait();
  const int t = blockIdx.x, tid = threadIdx.x;
  for (int i = tid; i < a.A; i += blockDim.x) {
    const float v = a.x[static_cast<size_t>(t) * a.A + i];
    xs[i] = a.round_bf16 ? __bfloat162float(__float2bfloat16_rn(v)) : v;
  }
  __syncthreads();
  const int nmb = (a.D + BM - 1) / BM;
  for (int m = 0; m < nmb; ++m) {
    const int n = m * BM + tid;
    float hv = 0.f;
    if (n < a.D) {
      const float* wr = a.w_in + static_cast<size_t>(n) * a.A;
      float acc = 0.f;
      for (int i = 0; i < a.A; ++i) acc = fmaf(wr[i], xs[i], acc);
      hv = acc + a.b_in[n] + a.temb[n];
      a.h[static_cast<size_t>(t) * a.D + n] = hv;
    }
    float sq = hv * hv;
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if ((tid & 31) == 0) wpart[tid >> 5] = sq;
    __syncthreads();
    if (tid == 0) a.ssq[m * a.T_pad + t] = ((wpart[0] + wpart[1]) + wpart[2]) + wpart[3];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(128) k_final_tc(const __grid_constant__ FinalArgs a) {
  extern __shared__ float hn[];
  grid_dep_launch();
  grid_dep_wait();
  const int t = blockIdx.x, tid = threadIdx.x;
  float ss = 0.f;
  for (int p = 0; p < a.ssq_parts; ++p) ss += a.ssq[p * a.T_pad + t];
  const float r = 1.0f / sqrtf(ss / a.D + a.eps);
  for (int k = tid; k < a.D; k += blockDim.x)
    hn[k] = __bfloat162float(__float2bfloat16_rn(a.h[static_cast<size_t>(t) * a.D + k] * r * a.g_f[k]));
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  for (int i = warp; i < a.A; i += nw) {
    const float* wr = a.w_out + static_cast<size_t>(i) * a.D;
    float acc = 0.f;
    for (int k = lane; k < a.D; k += 32) acc = fmaf(wr[k], hn[k], acc);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const size_t xi = static_cast<size_t>(t) * a.A + i;
      a.x_out[xi] = a.x_in[xi] + a.dt * (acc + a.b_out[i]);
    }
  }
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

}  // namespace

size_t gemm_smem_bytes(int Nt, int stages) {
  const size_t ring = static_cast<size_t>(stages) * (BM * KCB + static_cast<size_t>(Nt) * KCB);
  const size_t red = static_cast<size_t>(Nt) * RED_LD * sizeof(float);
  return ring > red ? ring : red;
}

size_t attn_smem_bytes(int H, int dh, int KC) {
  const int Hp = (H + 15) & ~15;
  const size_t qkv = (static_cast<size_t>(Hp) + 2 * KC) * (dh + ATT_PAD) * 2;
  const size_t obuf = static_cast<size_t>(Hp) * dh * 4 + static_cast<size_t>(Hp) * (dh + ATT_PAD) * 2;
  return qkv > obuf ? qkv : obuf;
}

cudaError_t tc_kernels_init() {
  cudaError_t e;
  int dev = 0, optin = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const void* fns[] = {reinterpret_cast<const void*>(k_gemm_tc), reinterpret_cast<const void*>(k_attn_tc<64>),
                       reinterpret_cast<const void*>(k_attn_tc<128>), reinterpret_cast<const void*>(k_attn_tc<256>)};
  for (const void* f : fns) {
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, f)) != cudaSuccess) return e;
    const int dyn = optin - static_cast<int>(fa.sharedSizeBytes);
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int max_dynamic_smem() {
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa;
  cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(k_gemm_tc));
  return optin - static_cast<int>(fa.sharedSizeBytes);
}

cudaError_t launch_gemm_tc(const GemmArgs& a, int n_tiles, cudaStream_t s, bool pdl) {
  GemmArgs copy = a;
  void* args[] = {&copy};
  return launch_ex(reinterpret_cast<const void*>(k_gemm_tc), dim3(a.S, a.MB, n_tiles), dim3(GEMM_THREADS),
                   gemm_smem_bytes(a.Nt, a.stages), s, pdl, a.S, args);
}

cudaError_t launch_attention_tc(const AttnArgs& a, int B, cudaStream_t s, bool pdl) {
  AttnArgs copy = a;
  void* args[] = {&copy};
  const int Hp = (a.H + 15) & ~15;
  const int nw = min(8, max(4, Hp / 16));
  const void* f = a.dh == 64 ? reinterpret_cast<const void*>(k_attn_tc<64>)
                : a.dh == 128 ? reinterpret_cast<const void*>(k_attn_tc<128>)
                              : reinterpret_cast<const void*>(k_attn_tc<256>);
  return launch_ex(f, dim3(a.C, a.Hq, B), dim3(32 * nw), attn_smem_bytes(a.H, a.dh, a.KC), s, pdl, a.C, args);
}

cudaError_t launch_inproj_tc(const InprojArgs& a, cudaStream_t s, bool pdl) {
  InprojArgs copy = a;
  void* args[] = {&copy};
  return launch_ex(reinterpret_cast<const void*>(k_inproj_tc), dim3(a.T), dim3(128), a.A * sizeof(float), s, pdl, 1,
                   args);
}

cudaError_t launch_final_tc(const FinalArgs& a, cudaStream_t s, bool pdl) {
  FinalArgs copy = a;
  void* args[] = {&copy};
  return launch_ex(reinterpret_cast<const void*>(k_final_tc), dim3(a.T), dim3(128), a.D * sizeof(float), s, pdl, 1,
                   args);
}

const void* inproj_kernel_ptr() { return reinterpret_cast<const void*>(k_inproj_tc); }
const void* final_kernel_ptr() { return reinterpret_cast<const void*>(k_final_tc); }

}  // namespace tc
}  // namespace fr
