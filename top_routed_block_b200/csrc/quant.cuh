// quant.cuh -- internal interface of the e4m3 block quantizer (quant.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fvattn {

// X bf16 [BH, N, d] (d % 8 == 0, 16-byte aligned) -> out e4m3 codes [BH, N, d],
// scale_exp int32 [BH, ceil(N / bs)].
cudaError_t launch_quant_e4m3(const void *X, int64_t BH, int N, int d, int bs, uint8_t *out, int32_t *scale_exp,
                              cudaStream_t stream);

}  // namespace fvattn
