// Kernels of the tensor-core path and their launch arguments.
//
// One Euler step is a chain of kernels launched with programmatic dependent
// launch (PDL) inside a CUDA graph:
//   inproj -> per layer { qkv GEMM -> attention -> o GEMM -> gate|up GEMM -> down GEMM } -> final
// Every GEMM kernel streams its weight slice into shared memory by bulk copy
// before it waits on its predecessor (weights do not depend on activations),
// so the weight stream overlaps the previous kernel.  Split-K partial sums are
// reduced inside a thread-block cluster through distributed shared memory in a
// fixed order (deterministic).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace fr {
namespace tc {

constexpr int BM = 128;            // output features per GEMM tile (tcgen05 M)
constexpr int KCB = 128;           // bytes of K per pipeline chunk (64 bf16 / 128 e4m3)
constexpr int MAX_STAGES = 8;      // ring slots per CTA
constexpr int GEMM_THREADS = 256;  // warp 0: weight producer, warp 1: MMA issuer, warps 2-7: B staging,
                                   // warps 4-7 also read TMEM in the epilogue
constexpr int NT_MAX = 256;        // tokens per tile (tcgen05 N)
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // a bounded wait gives up after 2 s

enum BKind : int { B_NORM = 0, B_ROWS = 1 };
enum EpiKind : int { EPI_QKV = 0, EPI_RESID = 1, EPI_GELU = 2 };

// Status word layout: [0] flags, [1] where, [2] block, [3] spare (see fr_sync_status).
enum : uint32_t { ST_TIMEOUT_BIT = 1u };

struct GemmArgs {
  // A operand: weights pre-tiled by the packer, [MB][NKC][BM rows x KCB bytes] core-matrix slabs
  const uint8_t* W;
  int MB, NKC;             // m-blocks, k-chunks
  int Nout;                // valid output rows (features) over all m-blocks
  int S;                   // split-K factor = cluster size along x
  int fp8;                 // 1: e4m3 operands (kind::f8f6f4), 0: bf16 (kind::f16)
  int stages;              // ring slots
  // token tiling
  int T;                   // valid tokens (B * H)
  int Nt;                  // tokens per n-tile (multiple of 16)
  // B operand source
  int b_kind;
  int Kdim;                // valid K elements
  const float* h;          // B_NORM: residual stream [T][D] fp32
  const float* gamma;      // B_NORM: RMSNorm gain [D]
  const float* ssq;        // B_NORM: per-token sum-of-squares partials [ssq_parts][T_pad]
  int ssq_parts;
  float eps;
  const float* s_a;        // fp8: activation scale of this projection input (device scalar)
  const uint8_t* act;      // B_ROWS: row-major [T][act_ld] bf16 or e4m3 bytes
  int act_ld;              // elements per row
  // epilogue
  int epi;
  const float* alpha;      // fp8: dequantisation scale s_a * s_w (device scalar), else nullptr
  int T_pad;               // row stride of ssq buffers
  // EPI_QKV
  __nv_bfloat16* q_out;    // [B][Hq][H][dh]
  __nv_bfloat16* kv_k;     // layer slice of the KV cache [B_max][Hkv][S_max][dh]
  __nv_bfloat16* kv_v;
  const float* rope_cos;   // [S_max][dh/2]
  const float* rope_sin;
  int H, P, S_max, Hq, Hkv, dh, MB_rot;
  // EPI_RESID
  float* h_out;            // [T][D] (+=)
  float* ssq_out;          // [MB][T_pad]
  int D;
  // EPI_GELU
  uint8_t* u_out;          // [T][F] bf16 or e4m3 bytes
  const float* s_a_out;    // fp8: scale of the down-projection input
  int F;
  unsigned* status;
};

struct AttnArgs {
  const __nv_bfloat16* q;      // [B][Hq][H][dh]
  const __nv_bfloat16* kv_k;   // layer slice [B_max][Hkv][S_max][dh]
  const __nv_bfloat16* kv_v;
  uint8_t* o;                  // [T][Hq*dh] bf16 or e4m3 bytes
  const float* s_a;            // fp8: scale of the O-projection input
  int fp8;
  int H, P, S_max, Hq, Hkv, dh;
  int C;                       // key chunks = cluster size
  int KC;                      // keys per chunk (multiple of 16)
  float scale;                 // 1/sqrt(dh)
};

struct InprojArgs {
  const float* x;              // [T][A] state at the start of the step
  const float* w_in;           // [D][A]
  const float* b_in;
  const float* temb;           // [D] of this step
  float* h;                    // [T][D]
  float* ssq;                  // [D/128][T_pad]
  int T, D, A, T_pad, round_bf16;
  int first;                   // marks the first kernel of a call (graph node lookup)
};

struct FinalArgs {
  const float* h;
  const float* ssq;            // [ssq_parts][T_pad]
  int ssq_parts;
  const float* g_f;
  const float* w_out;          // [A][D]
  const float* b_out;
  const float* x_in;           // [T][A]
  float* x_out;
  int T, D, A, T_pad;
  float eps, dt;
  int first;                   // x_in is the caller's x0 (graph node lookup)
  int last;                    // x_out is the caller's output (graph node lookup)
};

// Launchers (tc_kernels.cu).  `pdl` adds the programmatic-stream-serialisation attribute.
cudaError_t launch_gemm_tc(const GemmArgs& a, int n_tiles, cudaStream_t s, bool pdl);
cudaError_t launch_attention_tc(const AttnArgs& a, int B, cudaStream_t s, bool pdl);
cudaError_t launch_inproj_tc(const InprojArgs& a, cudaStream_t s, bool pdl);
cudaError_t launch_final_tc(const FinalArgs& a, cudaStream_t s, bool pdl);
size_t gemm_smem_bytes(int Nt, int stages);
size_t attn_smem_bytes(int H, int dh, int KC);
const void* inproj_kernel_ptr();
const void* final_kernel_ptr();
cudaError_t tc_kernels_init();    // function attributes (smem opt-in, non-portable clusters)
int max_dynamic_smem();            // dynamic shared memory a GEMM CTA may use
constexpr int ATTN_SUBK = 64;      // the attention key chunk is a multiple of this

}  // namespace tc
}  // namespace fr
