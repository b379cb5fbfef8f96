// Tensor-core kernel set: not built yet; every handle uses the stepwise kernels.
#include "internal.h"
#include "tensor_path.h"

namespace fr {

struct TensorPath {};

bool tensor_path_supports(const fr_config&) { return false; }
const char* tensor_path_limits() { return "tensor-core path not available"; }
size_t tensor_path_bytes(const fr_config&) { return 0; }
int tensor_path_create(const fr_config&, const TensorPathBuffers&, TensorPath**) { return FR_ERR_UNSUPPORTED; }
int tensor_path_pack_layer(TensorPath*, int, const fr_layer_weights&, const double*) { return FR_ERR_UNSUPPORTED; }
int tensor_path_finish_load(TensorPath*, cudaStream_t) { return FR_ERR_UNSUPPORTED; }
int tensor_path_set_scales(TensorPath*, const float*, const float*) { return FR_ERR_UNSUPPORTED; }
int tensor_path_denoise(TensorPath*, const float*, float*, int, int, cudaStream_t) { return FR_ERR_UNSUPPORTED; }
int tensor_path_launches(const TensorPath*, int) { return 0; }
void tensor_path_destroy(TensorPath*) {}

}  // namespace fr
