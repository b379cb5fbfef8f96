// Host side of the tensor-core path: weight pre-tiling, launch plan, CUDA-graph capture.
//
// Prior art and what changes here: the PhyAI page (optimisation paragraph) replays the
// ten-step Euler iteration of π0.5 from a CUDA graph and fuses the Q/K/V and gate/up
// projections; the FlashRT walkthrough (component 7) captures a pointer-only forward.
// This path captures every kernel of one call (K steps x L layers) into one graph whose
// kernels are chained by programmatic dependent launch, so each GEMM kernel streams
// its weights while its predecessor is still running.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <utility>
#include <vector>

#include "internal.h"
#include "persistent.h"
#include "tc_kernels.h"
#include "tensor_path.h"

namespace fr {

using namespace fr::tc;

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

struct ProjLayout {
  int rows = 0;      // output rows after permutation (padded to MB*BM)
  int K = 0;         // input features
  int MB = 0, NKC = 0;
  int NG = 0;        // w4: scale groups of 128 inputs
  size_t sc_off = 0; // w4: byte offset of the scales after the 4-bit codes
  size_t bytes = 0;  // tiled bytes per layer
};

// bf16 / e4m3: [MB][NKC][128 rows x 128 B] core-matrix slabs.  w4 (chunks of 64 inputs, as bf16):
// codes [MB][NKC][8 slabs][128 rows][4 B], then bf16 scales [MB][NG][128 rows].
ProjLayout make_layout(int rows, int K, int elem, int w4) {
  ProjLayout p;
  p.rows = rows;
  p.K = K;
  p.MB = ceil_div(rows, BM);
  p.NKC = ceil_div(K * elem, KCB);
  if (w4) {
    p.NG = ceil_div(p.NKC, 2);
    p.sc_off = static_cast<size_t>(p.MB) * p.NKC * (BM * KCB / 4);
    p.bytes = align_up(p.sc_off + static_cast<size_t>(p.MB) * p.NG * BM * 2, 1024);
  } else {
    p.bytes = static_cast<size_t>(p.MB) * p.NKC * BM * KCB;
  }
  return p;
}

struct GemmPlan {
  int S = 1, stages = 1;
  int red_tok = 0;   // S == 1: tokens per epilogue staging pass (0: the whole tile)
  int persist = 0;   // the persistent gate|up kernel
  int kpu = 1;       // k-chunks per ring slot
};

struct StepPlan {
  int B = 0, P = 0, H = 0, T = 0, NT = 0, Nt = 0;   // H: query tokens per sample (action rows or prefix tokens)
  GemmPlan qkv, o, gu, dn;
  int attn_C = 1, attn_KC = 64, attn_umma = 0;
};

struct RetargetNode {
  cudaGraphNode_t node = nullptr;   // node of the captured graph (kept alive with the exec)
  cudaKernelNodeParams kp{};
  bool is_inproj = false;
  InprojArgs ia{};
  FinalArgs fa{};
};

struct GraphEntry {
  cudaGraph_t graph = nullptr;      // owns the node handles used to retarget the exec
  cudaGraphExec_t exec = nullptr;
  std::vector<RetargetNode> nodes;  // kernels reading the caller's x0 or writing the caller's x_out
  const float* x0 = nullptr;
  float* x_out = nullptr;
  StepPlan plan;
  unsigned long long last_use = 0;  // graph-variant table: least recently used goes first
};

}  // namespace

struct TensorPath {
  fr_config c{};
  TensorPathBuffers tb{};
  int nsm = 148;
  int max_dyn = 0;
  int max_dyn2 = 0;              // dynamic shared memory of a GEMM CTA when two share an SM
  int fp8 = 0, elem = 2;
  int w4 = 0;                    // 4-bit weights dequantised in the GEMM (activations as bf16)
  int T_max = 0, T_pad = 0, MBd = 0, MB_rot = 0;
  int KB = 0;                    // 64-feature blocks of h per n-tile (D rounded up to 128)
  int ssq_ld = 0;                // columns of the Σh² partials (MBd rounded up to 4)
  int tok_alloc = 0;             // token rows of the tiled buffers (covers NT * Nt for every batch)
  ProjLayout qkv, o, gu, dn;
  size_t layer_bytes = 0;
  uint8_t* w = nullptr;          // [L][qkv|o|gu|dn] tiled weights
  float* gains = nullptr;        // [L][2][D]
  float* h = nullptr;            // tiled [NT][KB][Nt][64]
  float* ssq_a = nullptr;        // [T_pad][ssq_ld]
  float* ssq_b = nullptr;
  __nv_bfloat16* qbuf = nullptr; // [B_max][Hq][H][dh]
  uint8_t* obuf = nullptr;       // tiled [NT][NKC_o][Nt x 128] bf16 / e4m3
  uint8_t* ubuf = nullptr;       // tiled [NT][NKC_u][Nt x 128]
  uint8_t* xbuf = nullptr;       // bf16: tiled bf16(h * gamma) of the next RMSNorm, [NT][NKC_x][Nt x 128]
  float* xscratch = nullptr;     // split-K / key-chunk exchange scratch (L2-resident), shared by all kernels
  size_t xscratch_bytes = 0;
  float* xs = nullptr;           // [T_max][A] state between steps
  __nv_bfloat16* w_in_bf = nullptr;   // [A][D]
  __nv_bfloat16* w_out_bf = nullptr;  // [A][D]
  __nv_bfloat16* emb = nullptr;       // prefix pass: the embedded tokens of the call [B_max][H][D]
  cudaStream_t cap = nullptr;
  std::map<std::pair<int, int>, GraphEntry> graphs;   // graph-variant table keyed by (B, P)
  size_t graph_capacity = 8;
  unsigned long long use_clock = 0;
  std::vector<float> gains_host;
  // persistent kernel (batch-1-sized calls)
  unsigned* pk_ctr = nullptr;    // its counters, zero between calls
  int exec_mode = FR_EXEC_AUTO;
  unsigned long long wait_limit_ns = 2000000000ull;
  std::map<std::pair<int, int>, int> pk_fits;   // (B, P) -> the kernel is resident on every SM (1) or not (0)
  DevExtents ext_limit{};        // checked builds: smaller extents declared by fr_debug_limit_extent (0: none)
};

namespace {

struct Carve {
  char* base;         // nullptr: only measure
  size_t off = 0;
  template <typename T>
  T* take(size_t count, size_t align = 256) {
    off = align_up(off, align);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

void layouts(const fr_config& c, int elem, int w4, ProjLayout& qkv, ProjLayout& o, ProjLayout& gu, ProjLayout& dn) {
  qkv = make_layout((c.Hq + 2 * c.Hkv) * c.dh, c.D, elem, w4);
  o = make_layout(c.D, c.Hq * c.dh, elem, w4);
  gu = make_layout(2 * c.F, c.D, elem, w4);
  dn = make_layout(c.D, c.F, elem, w4);
}

size_t carve_all(TensorPath* tp, char* base) {
  const fr_config& c = tp->c;
  Carve cv{base};
  tp->w = cv.take<uint8_t>(tp->layer_bytes * c.L, 1024);
  tp->gains = cv.take<float>(static_cast<size_t>(c.L) * 2 * c.D);
  tp->h = cv.take<float>(static_cast<size_t>(tp->tok_alloc) * tp->KB * 64);
  tp->ssq_a = cv.take<float>(static_cast<size_t>(tp->T_pad) * tp->ssq_ld);
  tp->ssq_b = cv.take<float>(static_cast<size_t>(tp->T_pad) * tp->ssq_ld);
  tp->qbuf = cv.take<__nv_bfloat16>(static_cast<size_t>(c.B_max) * c.Hq * c.H * c.dh);
  tp->obuf = cv.take<uint8_t>(static_cast<size_t>(tp->tok_alloc) * tp->o.NKC * KCB);
  tp->ubuf = cv.take<uint8_t>(static_cast<size_t>(tp->tok_alloc) * tp->dn.NKC * KCB);
  tp->xbuf = cv.take<uint8_t>(tp->fp8 ? 0 : static_cast<size_t>(tp->tok_alloc) * tp->qkv.NKC * KCB);
  tp->xs = cv.take<float>(static_cast<size_t>(tp->T_max) * c.A);
  tp->xscratch = cv.take<float>(tp->xscratch_bytes / sizeof(float) + 64);
  tp->w_in_bf = cv.take<__nv_bfloat16>(static_cast<size_t>(c.D) * c.A);
  tp->w_out_bf = cv.take<__nv_bfloat16>(static_cast<size_t>(c.A) * c.D);
  tp->emb = cv.take<__nv_bfloat16>(c.role == FR_ROLE_PREFIX ? static_cast<size_t>(tp->T_max) * c.D : 0);
  tp->pk_ctr = cv.take<unsigned>(pk::CTR_WORDS);
  return align_up(cv.off, 1024);
}

void init_sizes(TensorPath* tp, const fr_config& c) {
  tp->c = c;
  tp->fp8 = c.dtype == FR_DTYPE_FP8;
  tp->w4 = c.dtype == FR_DTYPE_W4A16;
  tp->elem = tp->fp8 ? 1 : 2;
  tp->T_max = c.B_max * c.H;
  tp->T_pad = static_cast<int>(align_up(tp->T_max, 16));
  tp->MBd = ceil_div(c.D, BM);
  tp->MB_rot = (c.Hq + c.Hkv) * c.dh / 2 / 64;
  tp->KB = ceil_div(c.D, BM) * 2;
  tp->ssq_ld = static_cast<int>(align_up(tp->MBd, 4));
  const int nt_max = ceil_div(tp->T_max, NT_MAX);
  tp->tok_alloc = tp->T_max + 32 * nt_max;   // n-tiles of a call: at most 2 * nt_max, each padded by < 16 tokens
  layouts(c, tp->elem, tp->w4, tp->qkv, tp->o, tp->gu, tp->dn);
  tp->layer_bytes = tp->qkv.bytes + tp->o.bytes + tp->gu.bytes + tp->dn.bytes;
}

// Split-K / ring choice for one projection.  Batch-1-like tiles (Nt <= 64) are latency-bound:
// at most one CTA per SM (so the next kernel's CTAs can become resident and prefetch their
// weights next to it) and at most half an SM's shared memory; the cost counts waves, the split-K
// exchange, and weight chunks that must stream after the dependency wait.  Wider tiles are
// throughput-bound: no split-K unless the tiles leave most SMs idle.
GemmPlan choose_plan(int tiles, int NKC, int Nt, int b_kind, int fp8, int w4, int epi, int H, int xb, int nsm,
                     int max_dyn, int max_dyn2) {
  GemmPlan best;
  // k-chunks per ring slot for split S: two when every rank's chunk count is even and the operands
  // arrive by bulk copy (not B_NORM, not 4-bit weights) -- one copy per operand and slot
  auto kpu_ok = [&](int S) { return b_kind == B_ROWS && !w4 && NKC % (2 * S) == 0; };
  auto smem_k = [&](int S, int stages, int chunks, int red_tok, int kpu) {
    return gemm_smem_bytes(Nt, stages, b_kind, fp8, S, chunks, w4, epi, H, xb, red_tok, kpu);
  };
  // two-chunk slots only where the ring still double-buffers (or holds the whole k-range at once)
  auto kpu_of = [&](int S, size_t limit) {
    if (!kpu_ok(S)) return 1;
    const int chunks = ceil_div(NKC, S), units = chunks / 2;
    int stages = std::min(units, MAX_STAGES);
    while (stages > 1 && smem_k(S, stages, chunks, Nt, 2) > limit) --stages;
    return (stages >= 2 || stages == units) && smem_k(S, stages, chunks, Nt, 2) <= limit ? 2 : 1;
  };
  if (Nt > 64) {
    // The bf16 gate|up projection with at least two tiles per SM: the persistent kernel (one CTA per
    // SM walks the tiles; the epilogue of one tile overlaps the MMAs of the next), deepest ring that fits.
    if (epi == EPI_GELU && !fp8 && !w4 && b_kind == B_ROWS && tiles >= 2 * nsm && NKC % 2 == 0) {
      int stages = std::min(NKC / 2, MAX_STAGES);   // ring slots of two k-chunks
      while (stages > 2 && pt_smem_bytes(Nt, stages) > static_cast<size_t>(max_dyn)) --stages;
      if (stages >= 2 && pt_smem_bytes(Nt, stages) <= static_cast<size_t>(max_dyn)) {
        best.S = 1;
        best.stages = stages;
        best.persist = 1;
        return best;
      }
    }
    // More than one wave of unsplit tiles: two CTAs per SM, so that one CTA's epilogue runs while
    // the other's MMAs do (a ring of at least two slots; the accumulator staged in passes of half
    // the tile when the whole tile does not fit).
    if (tiles > nsm && max_dyn2 > 0) {
      const int chunks = NKC;
      // two-chunk slots where two of them still fit half an SM, else one-chunk slots: two CTAs per SM
      // matter more than fewer copies
      for (int kpu : {kpu_ok(1) ? 2 : 1, 1}) {
        const int units = NKC / kpu;
        for (int red_tok : {Nt, static_cast<int>(align_up(ceil_div(Nt, 2), 16))}) {
          int stages = std::min(units, MAX_STAGES);
          auto sm = [&](int st) { return gemm_smem_bytes(Nt, st, b_kind, fp8, 1, chunks, w4, epi, H, xb, red_tok, kpu); };
          while (stages > 2 && sm(stages) > static_cast<size_t>(max_dyn2)) --stages;
          if (stages >= 2 && sm(stages) <= static_cast<size_t>(max_dyn2)) {
            best.S = 1;
            best.stages = stages;
            best.red_tok = red_tok;
            best.kpu = kpu;
            return best;
          }
        }
      }
    }
    // throughput-bound tiles: split K in two only when the tiles leave most SMs idle; fall back to
    // the other split when the preferred one does not fit shared memory
    const int pref = (tiles * 2 <= nsm && NKC >= 2) ? 2 : 1;
    for (int S : {pref, 3 - pref}) {
      if (S > NKC) continue;
      const int kpu = kpu_of(S, static_cast<size_t>(max_dyn));
      const int chunks = ceil_div(NKC, S), units = chunks / kpu;
      int stages = std::min(units, MAX_STAGES);
      while (stages > 1 && smem_k(S, stages, chunks, Nt, kpu) > static_cast<size_t>(max_dyn)) --stages;
      best.S = S;
      best.stages = stages;
      best.kpu = kpu;
      if (smem_k(S, stages, chunks, Nt, kpu) <= static_cast<size_t>(max_dyn)) return best;
    }
    return best;   // nothing fits: the launch reports it
  }
  // at most half an SM's shared memory, so that the next kernel's CTAs fit beside this one's
  const size_t cap = std::min<size_t>(static_cast<size_t>(max_dyn), max_dyn2 > 0 ? static_cast<size_t>(max_dyn2) : 110 * 1024);
  double best_cost = 1e30;
  for (int S = 1; S <= 16 && S <= NKC; ++S) {
    const int kpu = kpu_of(S, cap);
    const int chunks = ceil_div(NKC, S), units = chunks / kpu;   // slot fills per CTA
    int stages = std::min(units, MAX_STAGES);
    while (stages > 1 && smem_k(S, stages, chunks, Nt, kpu) > cap) --stages;
    if (smem_k(S, stages, chunks, Nt, kpu) > static_cast<size_t>(max_dyn)) continue;
    const int waves = ceil_div(tiles * S, nsm);
    // streamed slots after the dependency wait; the copies in the cost count k-chunks
    const double cost = waves * (1.0 + (S > 1 ? 1.0 : 0.0) + 0.3 * kpu * (units - stages) + 0.05 * chunks);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.S = S;
      best.stages = stages;
      best.kpu = kpu;
    }
  }
  return best;
}

// Plan of one call: B samples of H query tokens (the action rows, or the prefix pass's tokens)
// attending to P cached keys plus themselves.
StepPlan make_plan(const TensorPath* tp, int B, int P, int H) {
  const fr_config& c = tp->c;
  StepPlan p;
  p.B = B;
  p.P = P;
  p.H = H;
  p.T = B * H;
  const int norm_kind = tp->fp8 ? B_NORM : B_ROWS;   // bf16: the producer wrote bf16(h*gamma) already
  auto plan_gemms = [&](StepPlan& q) {
    q.qkv = choose_plan(tp->qkv.MB * q.NT, tp->qkv.NKC, q.Nt, norm_kind, tp->fp8, tp->w4, EPI_QKV, H, 0, tp->nsm,
                        tp->max_dyn, tp->max_dyn2);
    q.o = choose_plan(tp->o.MB * q.NT, tp->o.NKC, q.Nt, B_ROWS, tp->fp8, tp->w4, EPI_RESID, H, !tp->fp8, tp->nsm,
                      tp->max_dyn, tp->max_dyn2);
    q.gu = choose_plan(tp->gu.MB * q.NT, tp->gu.NKC, q.Nt, norm_kind, tp->fp8, tp->w4, EPI_GELU, H, 0, tp->nsm,
                       tp->max_dyn, tp->max_dyn2);
    q.dn = choose_plan(tp->dn.MB * q.NT, tp->dn.NKC, q.Nt, B_ROWS, tp->fp8, tp->w4, EPI_RESID, H, !tp->fp8, tp->nsm,
                       tp->max_dyn, tp->max_dyn2);
  };
  // Token tiling.  The fewest tiles of at most NT_MAX tokens, unless more tiles (up to twice as many,
  // at least 160 tokens each: narrower tiles read their operands from shared memory about as fast as
  // the tensor core consumes them) give the four GEMMs less work per SM: per GEMM, rounds of CTAs over
  // the SMs x tokens x k-chunks per CTA, plus a fixed cost per round (prologue, exchange, epilogue) of
  // 1800 token-chunks (about 2 us).  Batch-1-sized calls keep one tile.
  const int nt0 = ceil_div(p.T, NT_MAX);
  double best = 1e300;
  for (int NT = nt0; NT <= 2 * nt0; ++NT) {
    StepPlan q = p;
    q.NT = NT;
    q.Nt = static_cast<int>(align_up(ceil_div(q.T, NT), 16));
    if (NT > nt0 && (q.Nt < 160 || ceil_div(q.T, q.Nt) != NT)) continue;
    plan_gemms(q);
    if (nt0 == 1) {
      p = q;
      break;
    }
    const ProjLayout* L[4] = {&tp->qkv, &tp->o, &tp->gu, &tp->dn};
    const GemmPlan* G[4] = {&q.qkv, &q.o, &q.gu, &q.dn};
    double cost = 0;
    for (int i = 0; i < 4; ++i) {
      const int rounds = ceil_div(L[i]->MB * NT * G[i]->S, tp->nsm);
      cost += rounds * (static_cast<double>(q.Nt) * ceil_div(L[i]->NKC, G[i]->S) + 1800.0);
    }
    if (cost < best) {
      best = cost;
      p = q;
    }
  }
  // the warp-MMA attention kernel holds at most 128 query rows per head: longer sequences take tcgen05
  p.attn_umma = attn_plan(P + H, attn_tiles(B, c.Hq, c.Hkv, H), tp->nsm, p.attn_C, p.attn_KC, H > 128);
  return p;
}

StepPlan make_plan(const TensorPath* tp, int B, int P) { return make_plan(tp, B, P, tp->c.H); }

// Pre-tile rows of one projection: rowsrc(r) gives the float32 row r (length K) or nullptr (zero row).
template <typename RowFn>
void tile_projection(const ProjLayout& L, int elem, double scale, RowFn rowsrc, std::vector<uint8_t>& out) {
  out.assign(L.bytes, 0);
  const int Kb = L.NKC * KCB;   // padded row bytes
  std::vector<uint8_t> row(Kb);
  std::vector<float> zero_pad;
  for (int r = 0; r < L.MB * BM; ++r) {
    const float* src = rowsrc(r);
    std::fill(row.begin(), row.end(), 0);
    if (src) {
      if (elem == 2) fr_round_bf16(src, reinterpret_cast<uint16_t*>(row.data()), L.K);
      else fr_quantize_e4m3(src, row.data(), L.K, scale);
    }
    const int mb = r / BM, rr = r % BM;
    for (int kc = 0; kc < L.NKC; ++kc) {
      uint8_t* blk = out.data() + (static_cast<size_t>(mb) * L.NKC + kc) * BM * KCB;
      for (int j = 0; j < KCB / 16; ++j)
        std::memcpy(blk + j * BM * 16 + (rr / 8) * 128 + (rr % 8) * 16, row.data() + kc * KCB + j * 16, 16);
    }
  }
}

// 4-bit codes and scales of one projection (fr_quantize_w4 per source row, groups along K).
template <typename RowFn>
void tile_projection_w4(const ProjLayout& L, RowFn rowsrc, std::vector<uint8_t>& out) {
  out.assign(L.bytes, 0);
  std::vector<int8_t> q(L.K);
  std::vector<uint16_t> sb(L.NG);
  uint16_t* scales = reinterpret_cast<uint16_t*>(out.data() + L.sc_off);
  for (int r = 0; r < L.MB * BM; ++r) {
    const float* src = rowsrc(r);
    if (!src) continue;   // padding rows: zero codes, zero scales
    fr_quantize_w4(src, 1, L.K, q.data(), sb.data());
    const int mb = r / BM, rr = r % BM;
    for (int g = 0; g < L.NG; ++g) scales[(static_cast<size_t>(mb) * L.NG + g) * BM + rr] = sb[g];
    for (int k = 0; k < L.K; ++k) {
      const int kc = k / 64, j = (k % 64) / 8, e = k % 8;
      uint8_t* word = out.data() + ((static_cast<size_t>(mb) * L.NKC + kc) * 8 + j) * BM * 4 + rr * 4;
      word[e >> 1] |= static_cast<uint8_t>((static_cast<uint8_t>(q[k]) & 0xF) << (4 * (e & 1)));
    }
  }
}

// Extents of the buffers the kernels store into (checked builds verify every store against them).
DevExtents extents(const TensorPath* tp, int B) {
  const fr_config& c = tp->c;
  DevExtents e;
  e.h = static_cast<uint64_t>(tp->tok_alloc) * tp->KB * 64;
  e.q = static_cast<uint64_t>(c.B_max) * c.Hq * c.H * c.dh;
  e.kv = tp->tb.kv_layer_bytes / 2;
  e.xbuf = tp->fp8 ? 0 : static_cast<uint64_t>(tp->tok_alloc) * tp->qkv.NKC * KCB;
  e.obuf = static_cast<uint64_t>(tp->tok_alloc) * tp->o.NKC * KCB;
  e.ubuf = static_cast<uint64_t>(tp->tok_alloc) * tp->dn.NKC * KCB;
  e.ssq = static_cast<uint64_t>(tp->T_pad) * tp->ssq_ld;
  e.x = static_cast<uint64_t>(B) * c.H * c.A;
  const DevExtents& m = tp->ext_limit;
  auto lim = [](uint64_t& v, uint64_t l) { if (l && l < v) v = l; };
  lim(e.h, m.h);
  lim(e.q, m.q);
  lim(e.kv, m.kv);
  lim(e.xbuf, m.xbuf);
  lim(e.obuf, m.obuf);
  lim(e.ubuf, m.ubuf);
  lim(e.ssq, m.ssq);
  lim(e.x, m.x);
  return e;
}

GemmArgs base_args(const TensorPath* tp, const StepPlan& p, const ProjLayout& L, const GemmPlan& g, int layer,
                   size_t w_off) {
  const fr_config& c = tp->c;
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.W = tp->w + layer * tp->layer_bytes + w_off;
  a.MB = L.MB;
  a.NKC = L.NKC;
  a.Nout = L.rows;
  a.S = g.S;
  a.stages = g.stages;
  a.red_tok = g.red_tok > 0 ? g.red_tok : p.Nt;
  a.persist = g.persist;
  a.kpu = g.kpu;
  a.pt_nt = p.NT;
  a.pt_ctas = std::min(L.MB * p.NT, tp->nsm);
  a.fp8 = tp->fp8;
  a.w4 = tp->w4;
  a.Wscale = tp->w4 ? reinterpret_cast<const uint16_t*>(a.W + L.sc_off) : nullptr;
  a.T = p.T;
  a.Nt = p.Nt;
  a.KB = tp->KB;
  a.D = c.D;
  a.eps = c.eps;
  a.ssq_ld = tp->ssq_ld;
  a.ssq_parts = tp->MBd;
  a.xscratch = tp->xscratch;
  a.status = tp->tb.status;
  a.ext = extents(tp, p.B);
  return a;
}

// Per-layer vectors of one recorded layer: the two norms' gains, the gain of the next layer's first
// norm (nullptr after the last layer), and the adaptive-RMSNorm gates and folded shifts (nullptr
// without it).
struct LayerVectors {
  const float *g1, *g2, *g1_next;
  const float *gate1, *gate2, *bias_qkv, *bias_gu;
};

// One layer: QKV GEMM (+RoPE, K/V into the cache), attention, O GEMM + residual, gate|up GEMM,
// down GEMM + residual.  qkv_only: stop after the QKV GEMM (the prefix pass's last layer, whose
// keys and values are all that is needed).
int record_layer(TensorPath* tp, const StepPlan& p, int l, const LayerVectors& v, bool qkv_only, cudaStream_t s) {
  const fr_config& c = tp->c;
  const size_t o_off = tp->qkv.bytes, gu_off = o_off + tp->o.bytes, dn_off = gu_off + tp->gu.bytes;
  cudaError_t e;
  const float* sa = tp->tb.s_a ? tp->tb.s_a + l * PI_COUNT : nullptr;
  const float* al = tp->tb.alpha ? tp->tb.alpha + l * PI_COUNT : nullptr;
  __nv_bfloat16* kvk = reinterpret_cast<__nv_bfloat16*>(tp->tb.kv_k + l * tp->tb.kv_layer_bytes);
  __nv_bfloat16* kvv = reinterpret_cast<__nv_bfloat16*>(tp->tb.kv_v + l * tp->tb.kv_layer_bytes);
  // QKV: RMSNorm fused into the B staging, split + RoPE fused into the epilogue
  GemmArgs q = base_args(tp, p, tp->qkv, p.qkv, l, 0);
  if (tp->fp8) {
    q.b_kind = B_NORM;
  } else {
    q.b_kind = B_ROWS;
    q.act = tp->xbuf;
    q.rscale = 1;
  }
  q.h = tp->h;
  q.gamma = v.g1;
  q.ssq = tp->ssq_a;
  q.s_a = tp->fp8 ? sa + PI_QKV : nullptr;
  q.alpha = tp->fp8 ? al + PI_QKV : nullptr;
  q.epi = EPI_QKV;
  q.q_out = tp->qbuf;
  q.kv_k = kvk;
  q.kv_v = kvv;
  q.rope_cos = tp->tb.rope_cos;
  q.rope_sin = tp->tb.rope_sin;
  q.H = p.H;
  q.P = p.P;
  q.S_max = c.P_max + c.H;
  q.Hq = c.Hq;
  q.Hkv = c.Hkv;
  q.dh = c.dh;
  q.MB_rot = tp->MB_rot;
  q.bias = v.bias_qkv;
  if ((e = launch_gemm_tc(q, p.NT, s, true)) != cudaSuccess) return cuda_fail(e, "qkv GEMM launch");
  if (qkv_only) return FR_OK;
  // attention over [cached keys; the tokens themselves]
  AttnArgs at{};
  at.q = tp->qbuf;
  at.kv_k = kvk;
  at.kv_v = kvv;
  at.o = tp->obuf;
  at.Nt = p.Nt;
  at.NKC_o = tp->o.NKC;
  at.s_a = tp->fp8 ? sa + PI_O : nullptr;
  at.fp8 = tp->fp8;
  at.H = p.H;
  at.P = p.P;
  at.S_max = c.P_max + c.H;
  at.Hq = c.Hq;
  at.Hkv = c.Hkv;
  at.dh = c.dh;
  at.C = p.attn_C;
  at.KC = p.attn_KC;
  at.scale = 1.0f / std::sqrt(static_cast<float>(c.dh));
  at.xscratch = tp->xscratch;
  at.status = tp->tb.status;
  at.umma = p.attn_umma;
  at.o_extent = extents(tp, p.B).obuf;
  if ((e = launch_attention_tc(at, p.B, s, true)) != cudaSuccess) return cuda_fail(e, "attention launch");
  // O projection + residual (+ sum of squares for the pre-MLP norm)
  GemmArgs og = base_args(tp, p, tp->o, p.o, l, o_off);
  og.b_kind = B_ROWS;
  og.act = tp->obuf;
  og.alpha = tp->fp8 ? al + PI_O : nullptr;
  og.epi = EPI_RESID;
  og.h_out = tp->h;
  og.ssq_out = tp->ssq_b;
  og.xb_out = tp->fp8 ? nullptr : tp->xbuf;
  og.xb_gamma = v.g2;
  og.NKC_x = tp->qkv.NKC;
  og.gate = v.gate1;
  if ((e = launch_gemm_tc(og, p.NT, s, true)) != cudaSuccess) return cuda_fail(e, "o GEMM launch");
  // gate|up with RMSNorm fused, GeLU(gate)*up epilogue
  GemmArgs gg = base_args(tp, p, tp->gu, p.gu, l, gu_off);
  if (tp->fp8) {
    gg.b_kind = B_NORM;
  } else {
    gg.b_kind = B_ROWS;
    gg.act = tp->xbuf;
    gg.rscale = 1;
  }
  gg.h = tp->h;
  gg.gamma = v.g2;
  gg.ssq = tp->ssq_b;
  gg.s_a = tp->fp8 ? sa + PI_GU : nullptr;
  gg.alpha = tp->fp8 ? al + PI_GU : nullptr;
  gg.epi = EPI_GELU;
  gg.u_out = tp->ubuf;
  gg.NKC_u = tp->dn.NKC;
  gg.s_a_out = tp->fp8 ? sa + PI_DOWN : nullptr;
  gg.F = c.F;
  gg.bias = v.bias_gu;
  if ((e = launch_gemm_tc(gg, p.NT, s, true)) != cudaSuccess) return cuda_fail(e, "gate|up GEMM launch");
  // down projection + residual (+ sum of squares for the next norm)
  GemmArgs dg = base_args(tp, p, tp->dn, p.dn, l, dn_off);
  dg.b_kind = B_ROWS;
  dg.act = tp->ubuf;
  dg.alpha = tp->fp8 ? al + PI_DOWN : nullptr;
  dg.epi = EPI_RESID;
  dg.h_out = tp->h;
  dg.ssq_out = tp->ssq_a;
  dg.xb_out = (tp->fp8 || !v.g1_next) ? nullptr : tp->xbuf;
  dg.xb_gamma = v.g1_next;   // gamma1 of layer l+1
  dg.NKC_x = tp->qkv.NKC;
  dg.gate = v.gate2;
  if ((e = launch_gemm_tc(dg, p.NT, s, true)) != cudaSuccess) return cuda_fail(e, "down GEMM launch");
  return FR_OK;
}

// The first kernel of a call: h, its Σh² partials and bf16(h * gamma1) of layer 0, from the
// in-projected actions plus the step's time embedding, or from the prefix pass's embeddings.
InprojArgs inproj_args(const TensorPath* tp, const StepPlan& p, const float* x_in, const float* temb,
                       const float* gamma1, bool first) {
  const fr_config& c = tp->c;
  InprojArgs ia{};
  ia.max_ctas = 2 * tp->nsm;
  ia.x = x_in;
  ia.w_in = tp->w_in_bf;
  ia.b_in = tp->tb.b_in;
  ia.temb = temb;
  ia.h = tp->h;
  ia.ssq = tp->ssq_a;
  ia.T = p.T;
  ia.D = c.D;
  ia.A = c.A;
  ia.Nt = p.Nt;
  ia.KB = tp->KB;
  ia.ssq_ld = tp->ssq_ld;
  ia.xb = tp->fp8 ? nullptr : tp->xbuf;
  ia.xb_gamma = gamma1;
  ia.NKC_x = tp->qkv.NKC;
  ia.first = first;
  ia.status = tp->tb.status;
  return ia;
}

int record_call(TensorPath* tp, const StepPlan& p, const float* x0, float* x_out, cudaStream_t s) {
  const fr_config& c = tp->c;
  const float dt = static_cast<float>(-1.0 / c.K);
  const bool ada = c.adarms != 0;
  cudaError_t e;
  for (int k = 0; k < c.K; ++k) {
    const float* x_in = (k == 0) ? x0 : tp->xs;
    float* x_nx = (k == c.K - 1) ? x_out : tp->xs;
    // adaptive RMSNorm: this step's gain of norm n (0 pre-attention, 1 pre-MLP) of layer l, and its
    // (scale | shift | gate) row
    auto ada_gain = [&](int l, int n) { return tp->tb.ada_gain + ((static_cast<size_t>(k) * c.L + l) * 2 + n) * c.D; };
    auto ada_mod = [&](int l, int n) { return tp->tb.ada_mod + ((static_cast<size_t>(k) * c.L + l) * 2 + n) * 3 * c.D; };
    auto gain = [&](int l, int n) -> const float* {
      return ada ? ada_gain(l, n) : tp->gains + (static_cast<size_t>(l) * 2 + n) * c.D;
    };
    InprojArgs ia = inproj_args(tp, p, x_in, ada ? nullptr : tp->tb.temb + static_cast<size_t>(k) * c.D, gain(0, 0),
                                k == 0);
    if ((e = launch_inproj_tc(ia, s, true)) != cudaSuccess) return cuda_fail(e, "in-proj kernel launch");
    for (int l = 0; l < c.L; ++l) {
      LayerVectors v{};
      v.g1 = gain(l, 0);
      v.g2 = gain(l, 1);
      v.g1_next = (l + 1 < c.L) ? gain(l + 1, 0) : nullptr;
      if (ada) {
        v.gate1 = ada_mod(l, 0) + 2 * c.D;
        v.gate2 = ada_mod(l, 1) + 2 * c.D;
        v.bias_qkv = tp->tb.ada_cq + (static_cast<size_t>(k) * c.L + l) * (c.Hq + 2 * c.Hkv) * c.dh;
        v.bias_gu = tp->tb.ada_cg + (static_cast<size_t>(k) * c.L + l) * 2 * c.F;
      }
      int rc = record_layer(tp, p, l, v, false, s);
      if (rc) return rc;
    }
    FinalArgs fa{};
    fa.max_ctas = 2 * tp->nsm;
    fa.h = tp->h;
    fa.ssq = tp->ssq_a;
    fa.ssq_ld = tp->ssq_ld;
    fa.ssq_parts = tp->MBd;
    fa.g_f = ada ? tp->tb.ada_gainf + static_cast<size_t>(k) * c.D : tp->tb.g_f;
    fa.w_out = tp->w_out_bf;
    fa.b_out = ada ? tp->tb.ada_bout + static_cast<size_t>(k) * c.A : tp->tb.b_out;
    fa.x_in = x_in;
    fa.x_out = x_nx;
    fa.T = p.T;
    fa.D = c.D;
    fa.A = c.A;
    fa.Nt = p.Nt;
    fa.KB = tp->KB;
    fa.eps = c.eps;
    fa.dt = dt;
    fa.first = (k == 0);
    fa.last = (k == c.K - 1);
    fa.status = tp->tb.status;
    if ((e = launch_final_tc(fa, s, true)) != cudaSuccess) return cuda_fail(e, "final kernel launch");
  }
  return FR_OK;
}

// The prefix pass (one forward over the P = p.H embedded tokens of each sample, no cached keys):
// every layer's rotated K and its V land in this handle's KV cache, slots 0..P-1.
int record_prefill(TensorPath* tp, const StepPlan& p, cudaStream_t s) {
  const fr_config& c = tp->c;
  InprojArgs ia = inproj_args(tp, p, nullptr, nullptr, tp->gains, false);
  ia.emb = tp->emb;
  cudaError_t e;
  if ((e = launch_inproj_tc(ia, s, true)) != cudaSuccess) return cuda_fail(e, "embedding kernel launch");
  for (int l = 0; l < c.L; ++l) {
    LayerVectors v{};
    v.g1 = tp->gains + static_cast<size_t>(l) * 2 * c.D;
    v.g2 = v.g1 + c.D;
    v.g1_next = (l + 1 < c.L) ? v.g1 + 2 * c.D : nullptr;
    int rc = record_layer(tp, p, l, v, l == c.L - 1, s);
    if (rc) return rc;
  }
  return FR_OK;
}

// ------------------------------------------------------------------ persistent kernel plan

// Split-K factor of one projection in the persistent kernel: at most PK_MAX_B chunks (128 KB of weights)
// per unit, so that its activation chunks fit the B region in one copy and most of its weights are
// resident before they are needed; and more splits while they leave at least half the SMs to the
// other phases (measured at pi0.5 batch 1: splits 2, 8, 2, 8 for QKV, O, gate|up, down).
// FR_PK_SPLITS="q,o,gu,dn" overrides (tuning).
int pk_split(int pg, int MB, int NKC, int nsm) {
  if (const char* e = std::getenv("FR_PK_SPLITS")) {
    int v[4] = {0, 0, 0, 0};
    if (std::sscanf(e, "%d,%d,%d,%d", &v[0], &v[1], &v[2], &v[3]) == 4 && v[pg] >= 1) {
      int S = std::min(v[pg], NKC);
      while (ceil_div(NKC, S) > pk::PK_MAX_B) ++S;   // a unit's activation chunks fit its B region
      return S;
    }
  }
  int S = 1;
  while (ceil_div(NKC, S) > pk::PK_MAX_B) S *= 2;
  while (S * 2 <= NKC && MB * S * 2 <= nsm / 2) S *= 2;
  return std::min(S, NKC);
}

// Arguments of one persistent call, or false when the call's shape is outside the kernel's limits.
// scratch_needed: report the exchange scratch the call needs instead of checking the handle's.
bool make_pk_args(TensorPath* tp, int B, int P, const float* x0, float* x_out, pk::PkArgs& a,
                  size_t* scratch_needed = nullptr) {
  const fr_config& c = tp->c;
  if (c.role != FR_ROLE_EXPERT || c.dtype != FR_DTYPE_BF16 || c.adarms) return false;
  const int T = B * c.H;
  if (T > pk::PK_MAX_T || c.A > 64 || c.D > 4096 || B * c.Hq > pk::PK_MAX_HEADS) return false;
  std::memset(&a, 0, sizeof(a));
  a.L = c.L;
  a.K = c.K;
  a.D = c.D;
  a.Hq = c.Hq;
  a.Hkv = c.Hkv;
  a.dh = c.dh;
  a.F = c.F;
  a.A = c.A;
  a.H = c.H;
  a.P = P;
  a.S_max = c.P_max + c.H;
  a.B = B;
  a.T = T;
  a.Nt = static_cast<int>(align_up(T, 16));
  a.KB = tp->KB;
  a.MBd = tp->MBd;
  a.MB_rot = tp->MB_rot;
  a.ssq_ld = tp->ssq_ld;
  a.NKC_x = tp->qkv.NKC;
  a.NKC_o = tp->o.NKC;
  a.NKC_u = tp->dn.NKC;
  a.eps = c.eps;
  a.dt = static_cast<float>(-1.0 / c.K);
  a.scale = 1.0f / std::sqrt(static_cast<float>(c.dh));
  a.G = tp->nsm;
  attn_chunks(P + c.H, a.C, a.KC);
  if (a.C > pk::PK_MAX_C) return false;
  const ProjLayout* L[4] = {&tp->qkv, &tp->o, &tp->gu, &tp->dn};
  const size_t w_off[4] = {0, tp->qkv.bytes, tp->qkv.bytes + tp->o.bytes, tp->qkv.bytes + tp->o.bytes + tp->gu.bytes};
  const uint8_t* act[4] = {tp->xbuf, tp->obuf, tp->xbuf, tp->ubuf};
  int placed = 0, max_nk = 1;
  size_t slices = 0, scratch = 0;
  for (int pg = 0; pg < 4; ++pg) {
    pk::PkGemm& g = a.g[pg];
    g.MB = L[pg]->MB;
    g.NKC = L[pg]->NKC;
    if (g.MB > pk::PK_MAX_MB) return false;
    g.S = pk_split(pg, g.MB, g.NKC, a.G);
    g.units = g.MB * g.S;
    g.w_off = w_off[pg];
    g.act = act[pg];
    g.base = placed % a.G;   // consecutive phases on consecutive CTAs: spreads the weight bytes per CTA
    placed += g.units;
    max_nk = std::max(max_nk, ceil_div(g.NKC, g.S));
    if (g.S > 1) {
      slices = std::max(slices, static_cast<size_t>(g.S) * ceil_div(a.Nt, g.S) * BM * 4);
      scratch = std::max(scratch, static_cast<size_t>(g.MB) * g.S * a.Nt * BM * 4);
    }
  }
  a.att_units = B * c.Hq * a.C;
  a.att_base = a.g[0].units % a.G;
  a.fi_base = placed % a.G;
  if (a.C > 1) scratch = std::max(scratch, attn_scratch_bytes(B, c.Hq, a.C, c.H, c.dh));
  if (scratch_needed) *scratch_needed = scratch;
  else if (scratch > tp->xscratch_bytes) return false;
  // shared memory: [weight ring | B region / epilogue stage | RoPE pairs or residual rows], attention over
  // the region after the ring
  a.nbs = std::min(pk::PK_MAX_B, max_nk);
  const size_t bring = static_cast<size_t>(a.nbs) * a.Nt * KCB;
  const size_t stage = std::max({bring, static_cast<size_t>(a.Nt) * RED_LD * 4, slices});
  const int cap = pk::pk_max_dynamic_smem();
  for (a.ring = pk::PK_MAX_RING; a.ring >= 2; --a.ring) {
    a.u_off = static_cast<uint32_t>(a.ring) * BM * KCB;
    a.rope_off = static_cast<uint32_t>(align_up(a.u_off + stage, 1024));
    a.hrow_off = a.rope_off;
    if (pk::pk_smem_bytes(a) <= static_cast<size_t>(cap)) break;
  }
  if (a.ring < 2) return false;
  a.W = tp->w;
  a.layer_bytes = tp->layer_bytes;
  a.gains = tp->gains;
  a.h = tp->h;
  a.ssq_a = tp->ssq_a;
  a.ssq_b = tp->ssq_b;
  a.q = tp->qbuf;
  a.obuf = tp->obuf;
  a.ubuf = tp->ubuf;
  a.xbuf = tp->xbuf;
  a.kv_k = reinterpret_cast<__nv_bfloat16*>(tp->tb.kv_k);
  a.kv_v = reinterpret_cast<__nv_bfloat16*>(tp->tb.kv_v);
  a.kv_layer_elems = tp->tb.kv_layer_bytes / sizeof(__nv_bfloat16);
  a.rope_cos = tp->tb.rope_cos;
  a.rope_sin = tp->tb.rope_sin;
  a.xscratch = tp->xscratch;
  a.x0 = x0;
  a.x_out = x_out;
  a.xs = tp->xs;
  a.temb = tp->tb.temb;
  a.w_in_t = tp->w_in_bf;
  a.b_in = tp->tb.b_in;
  a.w_out = tp->w_out_bf;
  a.b_out = tp->tb.b_out;
  a.g_f = tp->tb.g_f;
  a.ctr = tp->pk_ctr;
  a.status = tp->tb.status;
  a.flag_limit_ns = tp->wait_limit_ns;
  a.ext = extents(tp, B);
  return true;
}

// Whether a call of (B, P) runs the persistent kernel: its shape is within the kernel's limits and
// one CTA is resident on every SM.
bool pk_selected(TensorPath* tp, int B, int P, pk::PkArgs* out) {
  if (tp->exec_mode != FR_EXEC_PERSISTENT) return false;   // automatic choice: the CUDA graph
  pk::PkArgs a;
  if (!make_pk_args(tp, B, P, nullptr, nullptr, a)) return false;
  auto key = std::make_pair(B, P);
  auto it = tp->pk_fits.find(key);
  if (it == tp->pk_fits.end()) it = tp->pk_fits.emplace(key, pk::pk_max_blocks_per_sm(a) >= 1 ? 1 : 0).first;
  if (!it->second) return false;
  if (out) *out = a;
  return true;
}

int build_graph(TensorPath* tp, int B, int P, const float* x0, float* x_out, GraphEntry& ge) {
  const bool prefix = tp->c.role == FR_ROLE_PREFIX;   // (B, P): P prefix tokens per sample, no cached keys
  ge.plan = prefix ? make_plan(tp, B, 0, P) : make_plan(tp, B, P);
  cudaGraph_t g = nullptr;
  FR_CUDA(cudaStreamBeginCapture(tp->cap, cudaStreamCaptureModeThreadLocal));
  int rc = prefix ? record_prefill(tp, ge.plan, tp->cap) : record_call(tp, ge.plan, x0, x_out, tp->cap);
  cudaError_t e = cudaStreamEndCapture(tp->cap, &g);
  if (rc) {
    if (g) cudaGraphDestroy(g);
    return rc;
  }
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamEndCapture");
  ge.graph = g;
  size_t n = 0;
  FR_CUDA(cudaGraphGetNodes(g, nullptr, &n));
  std::vector<cudaGraphNode_t> nodes(n);
  FR_CUDA(cudaGraphGetNodes(g, nodes.data(), &n));
  e = cudaGraphInstantiate(&ge.exec, g, 0);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGraphInstantiate");
  for (cudaGraphNode_t nd : nodes) {
    cudaGraphNodeType t;
    FR_CUDA(cudaGraphNodeGetType(nd, &t));
    if (t != cudaGraphNodeTypeKernel) continue;
    cudaKernelNodeParams kp;
    FR_CUDA(cudaGraphKernelNodeGetParams(nd, &kp));
    RetargetNode rn;
    rn.node = nd;
    rn.kp = kp;
    if (kp.func == inproj_kernel_ptr()) {
      rn.ia = *static_cast<InprojArgs*>(kp.kernelParams[0]);
      if (!rn.ia.first) continue;
      rn.is_inproj = true;
    } else if (kp.func == final_kernel_ptr()) {
      rn.fa = *static_cast<FinalArgs*>(kp.kernelParams[0]);
      if (!rn.fa.first && !rn.fa.last) continue;
    } else {
      continue;
    }
    rn.kp.kernelParams = nullptr;
    rn.kp.extra = nullptr;
    ge.nodes.push_back(rn);
  }
  ge.x0 = x0;
  ge.x_out = x_out;
  return FR_OK;
}

// Point the graph's caller-facing nodes at this call's x0 / x_out.
int retarget(GraphEntry& ge, const float* x0, float* x_out) {
  if (ge.x0 == x0 && ge.x_out == x_out) return FR_OK;
  for (RetargetNode& rn : ge.nodes) {
    cudaKernelNodeParams kp = rn.kp;
    void* args[1];
    if (rn.is_inproj) {
      rn.ia.x = x0;
      args[0] = &rn.ia;
    } else {
      if (rn.fa.first) rn.fa.x_in = x0;
      if (rn.fa.last) rn.fa.x_out = x_out;
      args[0] = &rn.fa;
    }
    kp.kernelParams = args;
    FR_CUDA(cudaGraphExecKernelNodeSetParams(ge.exec, rn.node, &kp));
  }
  ge.x0 = x0;
  ge.x_out = x_out;
  return FR_OK;
}

}  // namespace

bool tensor_path_supports(const fr_config& c) {
  if (c.dtype != FR_DTYPE_BF16 && c.dtype != FR_DTYPE_FP8 && c.dtype != FR_DTYPE_W4A16) return false;
  if (c.dh != 64 && c.dh != 128 && c.dh != 256) return false;
  if (((c.Hq + c.Hkv) * c.dh / 2) % 64 != 0) return false;   // RoPE pairs fill whole m-blocks
  if ((c.Hkv * c.dh) % BM != 0) return false;                // V rows fill whole m-blocks
  if (c.F % 64 != 0) return false;                            // gate/up pairs fill whole m-blocks
  if (c.D % 16 != 0 || (c.Hq * c.dh) % 16 != 0) return false; // 16-byte operand rows
  if (c.D > 2048) return false;                               // per-token kernels keep a row in registers
  if (attn_smem_bytes(c.H, c.dh, 64, 1, 1) > 226 * 1024) return false;   // B200: 227 KB less the static part
  if (c.role == FR_ROLE_PREFIX) return c.dtype != FR_DTYPE_FP8;   // longer sequences: tcgen05 attention
  if (c.H > 128) return false;                                // one attention row-group pass per warp
  if (c.A > 64) return false;
  if (static_cast<size_t>(c.D) * c.A * 2 > 160 * 1024) return false;   // in/out-proj weights fit shared memory
  int C = 1, KC = 64;
  attn_chunks(c.P_max + c.H, C, KC);
  if (attn_smem_bytes(c.H, c.dh, KC, C, 0) > 200 * 1024) return false;
  return true;
}

// The launch plan of one call for a device of nsm SMs and the given dynamic shared-memory limits, on the
// host only (no device state): the token tiling, per projection (QKV, O, gate|up, down) the split, ring,
// staging pass, kernel, k-chunks per slot, shared memory, tiles and k-chunks, then the attention kernel
// and key split.  Returns the number of ints written.
int tensor_path_debug_plan(const fr_config& c, int B, int P, int nsm, int max_dyn, int max_dyn2, int* out, int n_out) {
  TensorPath tp;
  init_sizes(&tp, c);
  tp.nsm = nsm;
  tp.max_dyn = max_dyn;
  tp.max_dyn2 = max_dyn2;
  const StepPlan p = c.role == FR_ROLE_PREFIX ? make_plan(&tp, B, 0, P) : make_plan(&tp, B, P);
  std::vector<int> v = {p.NT, p.Nt};
  const ProjLayout* L[4] = {&tp.qkv, &tp.o, &tp.gu, &tp.dn};
  const GemmPlan* G[4] = {&p.qkv, &p.o, &p.gu, &p.dn};
  const int epi[4] = {EPI_QKV, EPI_RESID, EPI_GELU, EPI_RESID};
  for (int i = 0; i < 4; ++i) {
    const GemmPlan& g = *G[i];
    const int b_kind = (i == 0 || i == 2) && tp.fp8 ? B_NORM : B_ROWS;
    const int xb = (i == 1 || i == 3) && !tp.fp8;
    const size_t smem = g.persist ? pt_smem_bytes(p.Nt, g.stages)
                                  : gemm_smem_bytes(p.Nt, g.stages, b_kind, tp.fp8, g.S, ceil_div(L[i]->NKC, g.S), tp.w4,
                                                    epi[i], p.H, xb, g.red_tok > 0 ? g.red_tok : p.Nt, g.kpu);
    v.insert(v.end(), {g.S, g.stages, g.red_tok > 0 ? g.red_tok : p.Nt, g.persist, g.kpu, static_cast<int>(smem),
                       L[i]->MB * p.NT, L[i]->NKC});
  }
  v.insert(v.end(), {p.attn_umma, p.attn_C, p.attn_KC});
  const int n = static_cast<int>(v.size()) < n_out ? static_cast<int>(v.size()) : n_out;
  for (int i = 0; i < n; ++i) out[i] = v[i];
  return static_cast<int>(v.size());
}

const char* tensor_path_limits() {
  return "bf16/fp8/w4a16, dh in {64,128,256}, (Hq+Hkv)*dh/2 % 64 == 0, Hkv*dh % 128 == 0, F % 64 == 0, H <= 128, "
         "D % 16 == 0, D <= 2048, A <= 64, attention chunk fits shared memory";
}

// Exchange scratch needed by any batch size up to B_max and any prefix length up to P_max.
size_t exchange_scratch_bytes(TensorPath* tp) {
  const fr_config& c = tp->c;
  size_t mx = 0;
  // the persistent kernel's split-K partials at batch-1-sized calls (T <= 64 tokens in one tile); its
  // splits grow as its weight ring shrinks, and the ring is smallest at the longest prefix
  if (c.role == FR_ROLE_EXPERT)
    for (int B = 1; B <= c.B_max && B * c.H <= pk::PK_MAX_T; ++B) {
      pk::PkArgs a;
      size_t need = 0;
      if (make_pk_args(tp, B, c.P_max, nullptr, nullptr, a, &need)) mx = std::max(mx, need);
    }
  if (c.role == FR_ROLE_PREFIX) {   // every batch and prefix length the pass accepts (no cached keys)
    const ProjLayout* L[4] = {&tp->qkv, &tp->o, &tp->gu, &tp->dn};
    for (int B = 1; B <= c.B_max; ++B)
      for (int H = 1; H <= c.H; ++H) {
        const StepPlan p = make_plan(tp, B, 0, H);
        const GemmPlan* G[4] = {&p.qkv, &p.o, &p.gu, &p.dn};
        for (int i = 0; i < 4; ++i) mx = std::max(mx, gemm_scratch_bytes(p.NT, L[i]->MB, G[i]->S, p.Nt));
        if (p.attn_C > 1) mx = std::max(mx, attn_scratch_bytes(B, c.Hq, p.attn_C, H, c.dh));
      }
    return mx;
  }
  for (int B = 1; B <= c.B_max; ++B) {
    const StepPlan p = make_plan(tp, B, c.P_max);
    const ProjLayout* L[4] = {&tp->qkv, &tp->o, &tp->gu, &tp->dn};
    const GemmPlan* G[4] = {&p.qkv, &p.o, &p.gu, &p.dn};
    for (int i = 0; i < 4; ++i) mx = std::max(mx, gemm_scratch_bytes(p.NT, L[i]->MB, G[i]->S, p.Nt));
  }
  int cmax = 1;
  for (int P = 1; P <= c.P_max; ++P) {   // key chunks of every prefix length the handle accepts
    int C = 1, KC = 64;
    attn_chunks(P + c.H, C, KC);
    cmax = std::max(cmax, C);
  }
  mx = std::max(mx, attn_scratch_bytes(c.B_max, c.Hq, cmax, c.H, c.dh));
  return mx;
}

void device_params(TensorPath* tp) {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&tp->nsm, cudaDevAttrMultiProcessorCount, dev);
  tc_kernels_init();
  tp->max_dyn = max_dynamic_smem();
  tp->max_dyn2 = pair_dynamic_smem();
}

size_t tensor_path_bytes(const fr_config& c) {
  TensorPath tmp;
  init_sizes(&tmp, c);
  device_params(&tmp);
  tmp.xscratch_bytes = exchange_scratch_bytes(&tmp);
  return carve_all(&tmp, nullptr);
}

int tensor_path_create(const fr_config& c, const TensorPathBuffers& b, TensorPath** out) {
  TensorPath* tp = new TensorPath();
  init_sizes(tp, c);
  device_params(tp);
  tp->xscratch_bytes = exchange_scratch_bytes(tp);
  tp->tb = b;
  if (c.dtype != FR_DTYPE_FP8) {
    tp->tb.alpha = nullptr;
    tp->tb.s_a = nullptr;
  }
  if (carve_all(tp, b.base) > b.bytes) {
    delete tp;
    set_error("tensor path: buffer carve exceeds its allocation");
    return FR_ERR_CUDA;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&tp->nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = tc_kernels_init();
  if (e == cudaSuccess) e = pk::pk_init();
  if (e == cudaSuccess && tp->pk_ctr) e = cudaMemset(tp->pk_ctr, 0, pk::CTR_WORDS * sizeof(unsigned));
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&tp->cap, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    delete tp;
    return cuda_fail(e, "tensor path init");
  }
  tp->max_dyn = max_dynamic_smem();
  tp->max_dyn2 = pair_dynamic_smem();
  tp->gains_host.assign(static_cast<size_t>(c.L) * 2 * c.D, 1.f);
  *out = tp;
  return FR_OK;
}

int tensor_path_pack_layer(TensorPath* tp, int l, const fr_layer_weights& w, const double sw[4]) {
  const fr_config& c = tp->c;
  const int D = c.D, dh = c.dh, half = dh / 2, F = c.F;
  const int nq = c.Hq * dh, nk = c.Hkv * dh;
  std::vector<uint8_t> buf;
  uint8_t* dst = tp->w + l * tp->layer_bytes;
  // QKV rows: m-blocks of 64 rotate-half pairs (lo rows 0-63, hi rows 64-127), then V rows
  auto qkv_row = [&](int r) -> const float* {
    const int mb = r / BM, rr = r % BM;
    int cr;
    if (mb < tp->MB_rot) {
      const int pi = mb * 64 + (rr & 63);
      const int head = pi / half, j = pi % half;
      cr = head * dh + j + (rr >= 64 ? half : 0);
    } else {
      cr = nq + nk + (mb - tp->MB_rot) * BM + rr;
      if (cr >= nq + 2 * nk) return nullptr;
    }
    if (cr < nq) return w.wq + static_cast<size_t>(cr) * D;
    if (cr < nq + nk) return w.wk + static_cast<size_t>(cr - nq) * D;
    return w.wv + static_cast<size_t>(cr - nq - nk) * D;
  };
  if (tp->w4) tile_projection_w4(tp->qkv, qkv_row, buf);
  else tile_projection(tp->qkv, tp->elem, sw[PI_QKV], qkv_row, buf);
  FR_CUDA(cudaMemcpy(dst, buf.data(), buf.size(), cudaMemcpyHostToDevice));
  dst += tp->qkv.bytes;
  auto o_row = [&](int r) -> const float* { return r < D ? w.wo + static_cast<size_t>(r) * nq : nullptr; };
  if (tp->w4) tile_projection_w4(tp->o, o_row, buf);
  else tile_projection(tp->o, tp->elem, sw[PI_O], o_row, buf);
  FR_CUDA(cudaMemcpy(dst, buf.data(), buf.size(), cudaMemcpyHostToDevice));
  dst += tp->o.bytes;
  // gate|up rows: m-block mb holds gate features mb*64..+63 (rows 0-63) and the same up features (64-127)
  auto gu_row = [&](int r) -> const float* {
    const int mb = r / BM, rr = r % BM;
    const int f = mb * 64 + (rr & 63);
    if (f >= F) return nullptr;
    return (rr < 64 ? w.wg : w.wu) + static_cast<size_t>(f) * D;
  };
  if (tp->w4) tile_projection_w4(tp->gu, gu_row, buf);
  else tile_projection(tp->gu, tp->elem, sw[PI_GU], gu_row, buf);
  FR_CUDA(cudaMemcpy(dst, buf.data(), buf.size(), cudaMemcpyHostToDevice));
  dst += tp->gu.bytes;
  auto d_row = [&](int r) -> const float* { return r < D ? w.wd + static_cast<size_t>(r) * F : nullptr; };
  if (tp->w4) tile_projection_w4(tp->dn, d_row, buf);
  else tile_projection(tp->dn, tp->elem, sw[PI_DOWN], d_row, buf);
  FR_CUDA(cudaMemcpy(dst, buf.data(), buf.size(), cudaMemcpyHostToDevice));
  std::memcpy(&tp->gains_host[static_cast<size_t>(l) * 2 * D], w.g1, D * sizeof(float));
  std::memcpy(&tp->gains_host[static_cast<size_t>(l) * 2 * D + D], w.g2, D * sizeof(float));
  return FR_OK;
}

int tensor_path_finish_load(TensorPath* tp, cudaStream_t s) {
  const fr_config& c = tp->c;
  FR_CUDA(cudaMemcpy(tp->gains, tp->gains_host.data(), tp->gains_host.size() * 4, cudaMemcpyHostToDevice));
  // in/out-proj weights hold bf16-rounded values already: the conversion is exact
  FR_CUDA(launch_to_bf16_t(tp->tb.w_in, tp->w_in_bf, c.D, c.A, s));
  FR_CUDA(launch_to_bf16(tp->tb.w_out, tp->w_out_bf, static_cast<size_t>(c.A) * c.D, s));
  FR_CUDA(cudaStreamSynchronize(s));
  return FR_OK;
}

int tensor_path_set_scales(TensorPath*, const float*, const float*) {
  return FR_OK;   // kernels read the handle's device scale arrays directly
}

namespace {

void destroy_entry(GraphEntry& ge) {
  // an exec still running on a stream is freed by CUDA once it completes
  if (ge.exec) cudaGraphExecDestroy(ge.exec);
  if (ge.graph) cudaGraphDestroy(ge.graph);
  ge.exec = nullptr;
  ge.graph = nullptr;
}

// Drop least recently used variants until at most `keep` remain.
void evict_to(TensorPath* tp, size_t keep) {
  while (tp->graphs.size() > keep) {
    auto victim = tp->graphs.begin();
    for (auto it = tp->graphs.begin(); it != tp->graphs.end(); ++it)
      if (it->second.last_use < victim->second.last_use) victim = it;
    destroy_entry(victim->second);
    tp->graphs.erase(victim);
  }
}

}  // namespace

int tensor_path_set_graph_capacity(TensorPath* tp, int capacity) {
  tp->graph_capacity = static_cast<size_t>(capacity);
  evict_to(tp, tp->graph_capacity);
  return FR_OK;
}

int tensor_path_graph_count(const TensorPath* tp) { return static_cast<int>(tp->graphs.size()); }

int tensor_path_denoise(TensorPath* tp, const float* x0, float* x_out, int B, int P, cudaStream_t s) {
  pk::PkArgs pa;
  if (tp->c.role == FR_ROLE_EXPERT && pk_selected(tp, B, P, &pa)) {
    pa.x0 = x0;
    pa.x_out = x_out;
    FR_CUDA(pk::pk_launch(pa, s));
    return FR_OK;
  }
  if (tp->exec_mode == FR_EXEC_PERSISTENT && tp->c.role == FR_ROLE_EXPERT) {
    set_error("persistent execution: this call's shape is outside the persistent kernel's limits");
    return FR_ERR_UNSUPPORTED;
  }
  auto key = std::make_pair(B, P);
  auto it = tp->graphs.find(key);
  if (it == tp->graphs.end()) {
    evict_to(tp, tp->graph_capacity - 1);
    GraphEntry ge;
    int rc = build_graph(tp, B, P, x0, x_out, ge);
    if (rc) {
      if (ge.exec) cudaGraphExecDestroy(ge.exec);
      if (ge.graph) cudaGraphDestroy(ge.graph);
      return rc;
    }
    it = tp->graphs.emplace(key, ge).first;
  }
  it->second.last_use = ++tp->use_clock;
  int rc = retarget(it->second, x0, x_out);
  if (rc) return rc;
  FR_CUDA(cudaGraphLaunch(it->second.exec, s));
  return FR_OK;
}

int tensor_path_launches(TensorPath* tp, int B, int P) {
  if (tp->c.role == FR_ROLE_PREFIX) return 1 + 5 * (tp->c.L - 1) + 1;
  if (pk_selected(tp, B, P, nullptr)) return 1;
  return tp->c.K * (2 + 5 * tp->c.L);
}

int tensor_path_exec(TensorPath* tp, int B, int P) {
  if (tp->c.role != FR_ROLE_EXPERT) return FR_EXEC_GRAPH;
  return pk_selected(tp, B, P, nullptr) ? FR_EXEC_PERSISTENT : FR_EXEC_GRAPH;
}

int tensor_path_set_exec_mode(TensorPath* tp, int mode) {
  tp->exec_mode = mode;
  return FR_OK;
}

int tensor_path_limit_extent(TensorPath* tp, const char* name, unsigned long long elems) {
  DevExtents& m = tp->ext_limit;
  const struct { const char* n; uint64_t* v; } f[] = {{"h", &m.h},       {"q", &m.q},       {"kv", &m.kv},
                                                       {"xbuf", &m.xbuf}, {"obuf", &m.obuf}, {"ubuf", &m.ubuf},
                                                       {"ssq", &m.ssq},   {"x", &m.x}};
  for (const auto& e : f)
    if (std::strcmp(name, e.n) == 0) {
      *e.v = elems;
      evict_to(tp, 0);   // captured graphs carry the extents they were recorded with
      return FR_OK;
    }
  set_error("fr_debug_limit_extent: unknown buffer '%s' (h, q, kv, xbuf, obuf, ubuf, ssq, x)", name);
  return FR_ERR_ARG;
}

int tensor_path_set_wait_limit(TensorPath* tp, unsigned long long ns) {
  tp->wait_limit_ns = ns ? ns : 2000000000ull;
  return FR_OK;
}

int tensor_path_prefill(TensorPath* tp, const void* emb, int B, int P, cudaStream_t s) {
  FR_CUDA(cudaMemcpyAsync(tp->emb, emb, static_cast<size_t>(B) * P * tp->c.D * sizeof(__nv_bfloat16),
                          cudaMemcpyDeviceToDevice, s));
  return tensor_path_denoise(tp, nullptr, nullptr, B, P, s);   // the (B, P) graph of the pass
}

void tensor_path_destroy(TensorPath* tp) {
  if (!tp) return;
  for (auto& kv : tp->graphs) destroy_entry(kv.second);
  if (tp->cap) cudaStreamDestroy(tp->cap);
  delete tp;
}

}  // namespace fr
