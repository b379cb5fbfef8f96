// Tensor-core kernel set of the action-expert library (bf16 / fp8 handles).
#pragma once

#include <cuda_runtime.h>
#include <cstddef>

#include "fr.h"

namespace fr {

// Handle-owned buffers the tensor path reads or writes (carved in fr_create).
struct TensorPathBuffers {
  char* base;                 // tensor_path_bytes(cfg) bytes for the path's own buffers
  size_t bytes;
  const float* rope_cos;      // [S_max][dh/2]
  const float* rope_sin;
  char* kv_k;                 // [L][B_max][Hkv][S_max][dh] bf16
  char* kv_v;
  size_t kv_layer_bytes;
  float* x;                   // [B_max][H][A] state
  const float* temb;          // [K][D]
  const float* w_in;          // [D][A] (bf16-rounded values)
  const float* b_in;
  const float* w_out;         // [A][D]
  const float* b_out;
  const float* g_f;
  const float* alpha;         // [L][4] fp8 GEMM epilogue scales
  const float* s_a;           // [L][4] fp8 activation scales
  unsigned* status;           // device status word
  // adaptive RMSNorm (cfg.adarms), per Euler step k and layer l (see AdaRmsBuffers in runtime.cu)
  const float* ada_gain;      // [K][L][2][D] 1 + scale of the pre-attention / pre-MLP norm
  const float* ada_mod;       // [K][L][2][3D] (scale | shift | gate)
  const float* ada_gainf;     // [K][D] final norm gain
  const float* ada_bout;      // [K][A] b_out + W_out shift_f
  const float* ada_cq;        // [K][L][(Hq+2Hkv)dh] W_qkv shift_1
  const float* ada_cg;        // [K][L][2F] W_gu shift_2
};

struct TensorPath;

bool tensor_path_supports(const fr_config& c);
const char* tensor_path_limits();
int tensor_path_debug_plan(const fr_config& c, int B, int P, int nsm, int max_dyn, int max_dyn2, int* out, int n_out);
size_t tensor_path_bytes(const fr_config& c);
int tensor_path_create(const fr_config& c, const TensorPathBuffers& b, TensorPath** out);
int tensor_path_pack_layer(TensorPath* tp, int layer, const fr_layer_weights& w, const double sw[4]);
int tensor_path_finish_load(TensorPath* tp, cudaStream_t s);
int tensor_path_set_scales(TensorPath* tp, const float* s_a, const float* alpha);
int tensor_path_denoise(TensorPath* tp, const float* x0, float* x_out, int B, int P, cudaStream_t s);
int tensor_path_launches(TensorPath* tp, int B, int P);
int tensor_path_exec(TensorPath* tp, int B, int P);              // FR_EXEC_GRAPH or FR_EXEC_PERSISTENT
int tensor_path_set_exec_mode(TensorPath* tp, int mode);         // FR_EXEC_*
int tensor_path_set_wait_limit(TensorPath* tp, unsigned long long ns);
int tensor_path_limit_extent(TensorPath* tp, const char* name, unsigned long long elems);   // checked builds
// prefix-role paths: the pass over B x P embedded tokens (device bf16 [B][P][D]) into the KV cache
int tensor_path_prefill(TensorPath* tp, const void* emb, int B, int P, cudaStream_t s);
int tensor_path_set_graph_capacity(TensorPath* tp, int capacity);   // capacity >= 1
int tensor_path_graph_count(const TensorPath* tp);
void tensor_path_destroy(TensorPath* tp);

}  // namespace fr
