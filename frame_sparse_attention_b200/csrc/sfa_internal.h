// Host-side helpers shared by the libsfa translation units.
#pragma once

#include <cuda_runtime.h>

#include "sfa.h"

namespace sfa {

inline sfa_status cuda_status(cudaError_t e)
{
    return e == cudaSuccess ? SFA_OK : SFA_ERR_CUDA;
}

// launch errors (bad configuration, missing kernel image) surface here
inline sfa_status launch_status()
{
    return cuda_status(cudaGetLastError());
}

inline cudaStream_t as_cuda(sfa_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// k-way LSE merge of partials (sfa_merge.cu): slices [0, S) of o_part [S][rows][d] bf16
// and lse_part [S][rows] into o (strided as o_stride over [B][H][Lq]) and lse [rows];
// with o1 set, also slices [0, S1) into o1 (same strides) and lse1.  S <= d / 8.
sfa_status launch_lse_combine(int64_t rows, int S, int d, int H, int64_t Lq, const void *o_part,
                              const float *lse_part, void *o, const int64_t *o_stride, float *lse, cudaStream_t s,
                              int S1 = 0, void *o1 = nullptr, float *lse1 = nullptr);

}  // namespace sfa
