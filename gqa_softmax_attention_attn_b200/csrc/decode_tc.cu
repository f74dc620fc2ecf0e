// placeholder, replaced below
#include "kernels.h"
namespace attn_sink {
bool decode_bf16_supported(const DecodeShape &) { return false; }
cudaError_t launch_decode_bf16(const void *, const void *, const void *, const int *, const float *, void *,
                               float *, const DecodeShape &, float *, float *, cudaStream_t)
{
    return cudaErrorNotSupported;
}
}  // namespace attn_sink
