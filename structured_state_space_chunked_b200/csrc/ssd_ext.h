// ssd_ext.h -- feature maps and denominator normalisation (not part of the ABI).
#pragma once

#include "ssd_internal.h"

namespace ssd {

// dstate after feature map `kind` (SSD_FMAP_*) of an N-wide input; -1 if unknown
int fmap_dim(int kind, int N);
// dstB[r, :] = phi(srcB[r, :]) and dstC[r, :] = phi(srcC[r, :]) for rows r < rows; source
// rows N wide, mapped rows Nout wide
cudaError_t fmap_apply(int kind, int64_t rows, int N, int Nout, int bf16, const void* srcB, void* dstB,
                       const void* srcC, void* dstC, cudaStream_t stream);
// y[t, h, :] = y[t, h, :] / den[t, h] + D[h] x[t, h, :]
cudaError_t normalize_apply(int64_t T, int H, int P, int out_bf16, int in_bf16, void* y,
                            const float* den, const void* x, const float* D, cudaStream_t stream);

// the scan of a ones column, den[t, h] (fp32), zero state at each document's start.
// g is the problem with P = 1 and Q = kDenQ (its CUDA-core workspace, laid out by
// simt_carve_workspace, holds the chunk end/entering states); N up to 1024.
constexpr int kDenQ = 64;
bool den_scan_supported(int N);
cudaError_t den_scan(const Geom& g, const int32_t* cu, void* workspace, int* status, const void* dt,
                     const float* A, const float* dt_bias, const void* B, const void* C, float* den,
                     cudaStream_t stream);
// The tensor-core forward (ssd_tc.cu, N <= 128, 64-column units) with the division folded
// in: y = num / den + a.D x for a denominator den [tokens][H] computed beforehand.  The
// skip term enters the tile's mask diagonal as D den and each output row is scaled by
// 1 / den.  tc_den_supported says whether the shape and options take that kernel.
bool tc_den_supported(const Geom& g, const TcOpts& opts);
cudaError_t tc_forward_den(const Geom& g, const Args& a, const float* den, int* status, cudaStream_t stream,
                           int num_sms, const TcOpts& opts);
// the chunk table of packed documents (the CUDA-core forward's first kernel)
cudaError_t simt_varlen_table(const Geom& g, const int32_t* cu, const SimtWorkspace& ws, int* status,
                              cudaStream_t stream);

}  // namespace ssd
