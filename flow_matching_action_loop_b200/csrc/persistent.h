// Persistent, launch-free denoise kernel of the tensor-core path (batch-1-sized calls).
//
// One cooperative launch runs a whole fr_denoise call (K Euler steps x L layers): one CTA per
// SM, each CTA working through a fixed list of units of every phase
//   FI(-1) | for each step: for each layer { QKV, ATT, O, GU, DN } | FI(k)
// where FI(k) is the final norm + out-proj + Euler update of step k fused with the in-proj +
// time embedding of step k+1 (per token).  Phases hand over through global counters
// (release/acquire, bounded waits): a phase's units start when every unit of the phase before
// it has finished; the units of one split-K m-block or of one attention head exchange their
// partial results through an L2-resident scratch and are summed in a fixed order.
//
// Weights never wait on activations: warp 0 streams the weight chunks of every GEMM unit the
// CTA will run, in order, across phases, layers and steps, into a ring of shared-memory slots;
// the MMA warp consumes them as the activations arrive.  A CTA that finishes its unit of a
// phase therefore starts fetching its next unit's weights at once.
//
// PhyAI page, profiling paragraph: at batch 1 the action expert is a small share of the FLOPs
// but most of the latency, spent in many small launches; optimisation paragraph: the ten-step
// Euler iteration is replayed as one unit.  Here the unit is one kernel.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tc_kernels.h"

namespace fr {
namespace pk {

constexpr int PK_THREADS = 256;     // warp 0: weight producer, warp 1: MMA issuer, warps 4-7: workers
constexpr int PK_WORKERS = 128;
constexpr int PK_MAX_RING = 16;     // weight ring slots (16 KB each)
constexpr int PK_MAX_B = 8;         // activation (B operand) chunks of one unit (8 KB each at 64 tokens)
constexpr int PK_MAX_T = 64;        // tokens per call (one n-tile)
constexpr int PK_MAX_C = 16;        // attention key chunks per head

// GEMM phases in execution order (the attention phase sits between QKV and O)
enum : int { PG_QKV = 0, PG_O = 1, PG_GU = 2, PG_DN = 3 };

// Counter words (uint32), all zero between calls: the last CTA to leave a call clears them.
constexpr int CTR_DONE = 0;         // units finished, over the whole call (monotonic)
constexpr int CTR_ABORT = 1;        // set when a wait gave up: every CTA leaves its loops
constexpr int CTR_EXIT = 2;         // CTAs that have left
constexpr int PK_MAX_MB = 256;
constexpr int CTR_RED = 64;                              // [4][PK_MAX_MB] split-K partials landed
constexpr int PK_MAX_HEADS = 1024;
constexpr int CTR_ATT = CTR_RED + 4 * PK_MAX_MB;         // [B*Hq] key-chunk partials landed
constexpr int CTR_WORDS = CTR_ATT + PK_MAX_HEADS;

struct PkGemm {
  int MB, NKC, S;          // m-blocks, 64-element k-chunks, split-K factor
  int units, base;         // MB * S units; unit u runs on CTA (base + u) % G (and + G, ...)
  size_t w_off;            // byte offset of the projection inside one layer's tiled weights
  const uint8_t* act;      // B operand, tiled [NKC][Nt x 128 B]
};

struct PkArgs {
  int L, K, D, Hq, Hkv, dh, F, A, H, P, S_max, B, T, Nt, KB, MBd, MB_rot, ssq_ld, NKC_x, NKC_o, NKC_u;
  float eps, dt, scale;
  int G;                   // CTAs (one per SM, co-resident)
  int ring, nbs;           // weight ring slots, largest activation chunk count of a unit
  uint32_t u_off;          // shared memory: start of the region the workers' jobs share
  uint32_t rope_off;       // QKV units: (cos, sin) pairs of the m-block [H][64]
  uint32_t hrow_off;       // residual units: the owned tokens' h rows [2][TS][64]
  PkGemm g[4];
  int C, KC, att_units, att_base, fi_base;
  const uint8_t* W;        // tiled weights [L][qkv | o | gu | dn]
  size_t layer_bytes;
  const float* gains;      // [L][2][D]
  float* h;                // tiled [KB][Nt][64]
  float* ssq_a;            // [T_pad][ssq_ld]: written by DN / in-proj, read by QKV / final
  float* ssq_b;            // written by O, read by GU
  __nv_bfloat16* q;        // [B][Hq][H][dh]
  uint8_t* obuf;           // attention output, tiled [NKC_o][Nt x 128]
  uint8_t* ubuf;           // GeLU(gate) * up, tiled [NKC_u][Nt x 128]
  uint8_t* xbuf;           // bf16(h * gamma) of the next norm, tiled [NKC_x][Nt x 128]
  __nv_bfloat16* kv_k;     // [L][B_max][Hkv][S_max][dh]
  __nv_bfloat16* kv_v;
  size_t kv_layer_elems;
  const float* rope_cos;   // [S_max][dh/2]
  const float* rope_sin;
  float* xscratch;         // split-K / key-chunk partials
  const float* x0;         // [T][A]
  float* x_out;
  float* xs;               // [T][A] state between steps
  const float* temb;       // [K][D]
  const __nv_bfloat16* w_in_t;   // [A][D]
  const float* b_in;
  const __nv_bfloat16* w_out;    // [A][D]
  const float* b_out;
  const float* g_f;
  unsigned* ctr;           // CTR_WORDS counters
  unsigned* status;        // device status word
  unsigned long long flag_limit_ns;   // bound of every wait on another CTA
  tc::DevExtents ext;      // extents of the stored-to buffers (checked builds)
};

size_t pk_smem_bytes(const PkArgs& a);
cudaError_t pk_launch(const PkArgs& a, cudaStream_t s);
cudaError_t pk_init();                      // kernel attributes (once per device)
int pk_max_blocks_per_sm(const PkArgs& a);  // co-residency check (0 on error)
int pk_max_dynamic_smem();                  // dynamic shared memory one CTA of the kernel may use

}  // namespace pk
}  // namespace fr
