// Placeholder for the tensor-core kernels: reports every shape unsupported.
#include "tpa_tensor.h"

namespace tpa {
bool tensor_decode_supported(int, int, int, int, int) { return false; }
int tensor_decode_token_granule(int) { return 64; }
int tensor_decode_default_splits(int, int, int, int) { return 1; }
cudaError_t launch_tensor_decode(const TensorDecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }
bool tensor_prefill_supported(int, int, int, int, int, int) { return false; }
size_t tensor_prefill_workspace_bytes(int, int, int, int) { return 0; }
cudaError_t launch_tensor_prefill(const TensorPrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace tpa
