// Kernels of the tensor-core path and their launch arguments.
//
// One Euler step is a chain of kernels launched with programmatic dependent
// launch (PDL) inside a CUDA graph:
//   inproj -> per layer { qkv GEMM -> attention -> o GEMM -> gate|up GEMM -> down GEMM } -> final
// Every kernel fetches what does not depend on its predecessor (weights, prefix
// keys/values) before it waits on it, so those loads overlap the previous kernel.
// Loads on the dependent side are asynchronous bulk copies issued up front.  Split-K
// partial tiles and attention key-chunk partials are exchanged inside a thread-block
// cluster through an L2-resident scratch buffer (stored straight from registers, one
// cluster barrier with release/acquire semantics, then read by their owner CTA) and
// summed in rank order (deterministic).  On this part the L2 moves these partials
// several times faster than distributed shared memory does.
//
// Activation layouts (all per call, n-tile of Nt tokens, nt = t / Nt, r = t % Nt):
//   h (residual, fp32)   [NT][D/64][Nt][64]          -- a 64-feature chunk of an n-tile is contiguous
//   o, u (GEMM B inputs) [NT][NKC][Nt x 128 bytes]   -- the tcgen05 operand tile of one k-chunk, ready
//                                                       for one bulk copy (see btile_offset)
//   Σh² partials (fp32)  [T_pad][ssq_ld]             -- one 128-feature block per column, token-major
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace fr {
namespace tc {

constexpr int BM = 128;            // output features per GEMM tile (tcgen05 M)
constexpr int KCB = 128;           // bytes of K per pipeline chunk (64 bf16 / 128 e4m3)
constexpr int MAX_STAGES = 8;      // ring slots per CTA
constexpr int GEMM_THREADS = 256;  // warp 0: bulk-copy producer, warp 1: MMA issuer, warps 2-7: B conversion,
                                   // warps 4-7 also read TMEM in the epilogue
constexpr int NT_MAX = 256;        // tokens per tile (tcgen05 N)
constexpr int RED_LD = BM + 4;     // floats per token row of the epilogue exchange buffers
constexpr int ATTN_SUBK = 64;      // keys per online-softmax step; the attention key chunk is a multiple of it
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // a bounded wait gives up after 2 s

enum BKind : int { B_NORM = 0, B_ROWS = 1 };
enum EpiKind : int { EPI_QKV = 0, EPI_RESID = 1, EPI_GELU = 2 };

// Status word layout: [0] flags, [1] where, [2] block (see fr_sync_status).
enum : uint32_t { ST_TIMEOUT_BIT = 1u, ST_BOUNDS_BIT = 2u };

// Extents of the buffers the kernels store into (elements of the buffer's type; bytes for the
// tiled operand buffers).  Checked builds (-DFR_DEVICE_CHECKS) verify every epilogue store index
// against them; the product build carries them unused.
struct DevExtents {
  uint64_t h;      // tiled residual, floats
  uint64_t q;      // q buffer, bf16 elements
  uint64_t kv;     // one layer's K (or V) cache slice, bf16 elements
  uint64_t xbuf;   // bf16(h * gamma) operand, bytes
  uint64_t obuf;   // attention output operand, bytes
  uint64_t ubuf;   // GeLU(gate) * up operand, bytes
  uint64_t ssq;    // sums of squares, floats
  uint64_t x;      // action state of the call, floats
};

// Byte offset of element (row r of n-tile nt, K byte kb) in a tiled GEMM B input.
__host__ __device__ __forceinline__ size_t btile_offset_nt(int nt, int r, int kb, int Nt, int NKC) {
  const int kc = kb >> 7, w = kb & 127;
  return (static_cast<size_t>(nt) * NKC + kc) * Nt * 128 + (w >> 4) * Nt * 16 + (r >> 3) * 128 + (r & 7) * 16 +
         (w & 15);
}
// Byte offset of element (token t, K byte kb) in a tiled GEMM B input.
__host__ __device__ __forceinline__ size_t btile_offset(int t, int kb, int Nt, int NKC) {
  const int nt = t / Nt;
  return btile_offset_nt(nt, t - nt * Nt, kb, Nt, NKC);
}
// Float offset of element (row r of n-tile nt, feature f) in the tiled residual h.
__host__ __device__ __forceinline__ size_t htile_offset_nt(int nt, int r, int f, int Nt, int KB) {
  return ((static_cast<size_t>(nt) * KB + (f >> 6)) * Nt + r) * 64 + (f & 63);
}
// Float offset of element (token t, feature f) in the tiled residual h.
__host__ __device__ __forceinline__ size_t htile_offset(int t, int f, int Nt, int KB) {
  const int nt = t / Nt;
  return htile_offset_nt(nt, t - nt * Nt, f, Nt, KB);
}

struct GemmArgs {
  // A operand: weights pre-tiled by the packer, [MB][NKC][BM rows x KCB bytes] core-matrix slabs
  const uint8_t* W;           // w4: 4-bit codes [MB][NKC][8 slabs][128 rows][4 B] (8 codes per 4 B, low nibble first)
  const uint16_t* Wscale;     // w4: bf16 scales [MB][NG][128 rows], one per 128 inputs (two chunks)
  int w4;                     // 1: 4-bit weights, dequantised to bf16(q * s) in shared memory
  int MB, NKC;             // m-blocks, k-chunks
  int Nout;                // valid output rows (features) over all m-blocks
  int S;                   // split-K factor = cluster size along x
  int fp8;                 // 1: e4m3 operands (kind::f8f6f4), 0: bf16 (kind::f16)
  int stages;              // ring slots
  int T, Nt;               // valid tokens, tokens per n-tile (multiple of 16)
  int b_kind;
  // B_NORM: RMSNorm(+e4m3) of the residual h, converted in shared memory
  const float* h;          // tiled [NT][KB][Nt][64]
  int KB;                  // D / 64
  int D;
  const float* gamma;      // [D]
  const float* ssq;        // [T_pad][ssq_ld]
  int ssq_ld, ssq_parts;
  float eps;
  const float* s_a;        // fp8: activation scale of this projection input (device scalar)
  // B_ROWS: already-quantised activation in the tiled operand layout
  const uint8_t* act;      // [NT][NKC][Nt x 128]
  int rscale;              // 1: B_ROWS holds bf16(h*gamma); the epilogue scales token t by rstd_t (from ssq)
  // epilogue
  int epi;
  const float* alpha;      // fp8: dequantisation scale s_a * s_w (device scalar), else nullptr
  const float* bias;       // EPI_QKV / EPI_GELU: added per output feature (natural row order), or nullptr
  const float* gate;       // EPI_RESID: the update is scaled per feature before h +=, or nullptr
  // EPI_QKV
  __nv_bfloat16* q_out;    // [B][Hq][H][dh]
  __nv_bfloat16* kv_k;     // layer slice of the KV cache [B_max][Hkv][S_max][dh]
  __nv_bfloat16* kv_v;
  const float* rope_cos;   // [S_max][dh/2]
  const float* rope_sin;
  int H, P, S_max, Hq, Hkv, dh, MB_rot;
  // EPI_RESID
  float* h_out;            // tiled h (+=)
  float* ssq_out;          // [T_pad][ssq_ld], column mb
  uint8_t* xb_out;         // bf16(h_new * xb_gamma) in the tiled operand layout of the next norm's GEMM, or nullptr
  const float* xb_gamma;   // gain of the next RMSNorm
  int NKC_x;
  // EPI_GELU
  uint8_t* u_out;          // tiled [NT][NKC_u][Nt x 128]
  int NKC_u;
  const float* s_a_out;    // fp8: scale of the down-projection input
  int F;
  int red_tok;             // S == 1: tokens per epilogue staging pass (Nt, or fewer so that two CTAs share an SM)
  int kpu;                 // k-chunks per ring slot (1, or 2 without B_NORM / 4-bit weights when every rank's count is even)
  int persist;             // 1: the persistent gate|up kernel (one CTA per SM over the tiles; bf16, S == 1)
  int pt_ctas, pt_nt;      // persistent: CTAs of the launch, n-tiles
  // split-K exchange (S > 1): fp32 partial tiles [NT][MB][S][Nt][128], L2-resident scratch
  float* xscratch;
  unsigned* status;
  DevExtents ext;
};

struct AttnArgs {
  const __nv_bfloat16* q;      // [B][Hq][H][dh]
  const __nv_bfloat16* kv_k;   // layer slice [B_max][Hkv][S_max][dh]
  const __nv_bfloat16* kv_v;
  uint8_t* o;                  // tiled [NT][NKC_o][Nt x 128], bf16 or e4m3
  int Nt, NKC_o;
  const float* s_a;            // fp8: scale of the O-projection input
  int fp8;
  int H, P, S_max, Hq, Hkv, dh;
  int C;                       // key chunks = cluster size
  int KC;                      // keys per chunk (multiple of ATTN_SUBK)
  float scale;                 // 1/sqrt(dh)
  float* xscratch;             // C > 1: partial rows [B][Hq][C][H][dh + 4] (O, max, sum), L2-resident scratch
  int o_rowmajor;              // 1: o is bf16 [B][H][Hq*dh] row-major instead of the tiled operand layout
  unsigned* status;            // device status word (timeouts), or nullptr
  int umma;                    // 1: tcgen05 kernel over GQA-group tiles; 0: warp-MMA kernel per query head
  uint64_t o_extent;           // bytes of o (checked builds)
  // tcgen05 kernel: tensor maps of this layer's K and V ([B*Hkv][P+H][dh], planes S_max rows apart),
  // 128-byte swizzle; written by launch_attention_tc.  kv_boxes == 1: one box per 64-key sub-chunk
  // (64 features x 64 keys x dh/64 feature blocks, a 4-D view); otherwise dh/64 boxes of 64 x 64
  CUtensorMap tm_k, tm_v;
  int kv_boxes;
};

// Key chunks of the split-KV attention over S keys: at most 16 (one cluster), each a multiple
// of the 64-key sub-chunk.  This is the largest split; it sizes the merge scratch.
inline void attn_chunks(int S, int& C, int& KC) {
  C = S < 16 * ATTN_SUBK ? (S + ATTN_SUBK - 1) / ATTN_SUBK : 16;
  const int per = (S + C - 1) / C;
  KC = (per + ATTN_SUBK - 1) / ATTN_SUBK * ATTN_SUBK;
  C = (S + KC - 1) / KC;
}

// Query-row tiles of the attention kernel: 128 rows of (query head, action row) per KV head.
inline int attn_tiles(int B, int Hq, int Hkv, int H) { return B * Hkv * ((Hq / Hkv * H + 127) / 128); }

// Attention kernel and key split.  When even the largest split leaves SMs idle (batch-1 sizes)
// the warp-MMA kernel runs, one CTA per (key chunk, query head), with attn_chunks' split;
// otherwise the tcgen05 kernel runs with enough chunks to give every SM a CTA.  Either way
// C <= attn_chunks' C, so the scratch bound holds.  Returns 1 for the tcgen05 kernel.
inline int attn_plan(int S, int tiles, int nsm, int& C, int& KC, bool force_umma = false) {
  int cmax = 1, kc = 64;
  attn_chunks(S, cmax, kc);
  if (tiles * cmax < nsm && !force_umma) {
    C = cmax;
    KC = kc;
    return 0;
  }
  int want = nsm / (tiles > 0 ? tiles : 1);
  want = want < 1 ? 1 : (want > cmax ? cmax : want);
  const int per = (S + want - 1) / want;
  KC = (per + ATTN_SUBK - 1) / ATTN_SUBK * ATTN_SUBK;
  C = (S + KC - 1) / KC;
  return 1;
}

struct InprojArgs {
  int max_ctas;                // grid cap (tokens are strided over the CTAs); 0: one CTA per token
  const float* x;              // [T][A] state at the start of the step
  const __nv_bfloat16* w_in;   // [A][D] (transposed by the loader)
  const float* b_in;
  const float* temb;           // [D] of this step, or nullptr
  const __nv_bfloat16* emb;    // prefix pass: h = emb [T][D] (no in-proj, no time), or nullptr
  float* h;                    // tiled h
  float* ssq;                  // [T_pad][ssq_ld]
  uint8_t* xb;                 // bf16(h * gamma1 of layer 0), tiled operand layout, or nullptr
  const float* xb_gamma;
  int NKC_x;
  int T, D, A, Nt, KB, ssq_ld;
  int first;                   // x is the caller's x0 (graph node lookup)
  unsigned* status;            // device status word (timeouts), or nullptr
};

struct FinalArgs {
  int max_ctas;                // grid cap (tokens are strided over the CTAs); 0: one CTA per token
  const float* h;              // tiled h
  const float* ssq;            // [T_pad][ssq_ld]
  int ssq_ld, ssq_parts;
  const float* g_f;
  const __nv_bfloat16* w_out;  // [A][D]
  const float* b_out;
  const float* x_in;           // [T][A]
  float* x_out;
  int T, D, A, Nt, KB;
  float eps, dt;
  int first;                   // x_in is the caller's x0 (graph node lookup)
  int last;                    // x_out is the caller's output (graph node lookup)
  unsigned* status;            // device status word (timeouts), or nullptr
};

// Launchers (tc_kernels.cu).  `pdl` adds the programmatic-stream-serialisation attribute.
cudaError_t launch_gemm_tc(const GemmArgs& a, int n_tiles, cudaStream_t s, bool pdl);
cudaError_t launch_attention_tc(const AttnArgs& a, int B, cudaStream_t s, bool pdl);
cudaError_t launch_inproj_tc(const InprojArgs& a, cudaStream_t s, bool pdl);
cudaError_t launch_final_tc(const FinalArgs& a, cudaStream_t s, bool pdl);
cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, size_t n, cudaStream_t s);
cudaError_t launch_to_bf16_t(const float* src, __nv_bfloat16* dst, int rows, int cols, cudaStream_t s);
cudaError_t launch_wait_selftest(unsigned* status, unsigned long long limit_ns, cudaStream_t s);
size_t gemm_smem_bytes(int Nt, int stages, int b_kind, int fp8, int S, int nk, int w4, int epi, int H, int xb,
                       int red_tok, int kpu);
size_t gemm_scratch_bytes(int NT, int MB, int S, int Nt);
size_t attn_scratch_bytes(int B, int Hq, int C, int H, int dh);
size_t attn_smem_bytes(int H, int dh, int KC, int C, int umma);
const void* inproj_kernel_ptr();
const void* final_kernel_ptr();
cudaError_t tc_kernels_init();    // function attributes (smem opt-in, carveout, non-portable clusters)
int max_dynamic_smem();           // dynamic shared memory a GEMM CTA may use
int pair_dynamic_smem();          // dynamic shared memory of a GEMM CTA that shares its SM with another
size_t pt_smem_bytes(int Nt, int stages);   // dynamic shared memory of the persistent gate|up GEMM

}  // namespace tc
}  // namespace fr
