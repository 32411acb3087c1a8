// ssd_bwd.h -- declarations of the backward pass (not part of the ABI).
#pragma once

#include "ssd_internal.h"

namespace ssd {

// The CUDA-core forward stopped after its state pass: ws.cs, ws.delta, the state
// entering every chunk in ws.states, and a.final_states when given (y untouched).
cudaError_t simt_states(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                        cudaStream_t stream);
// the same in two parts around a chunk-state product of the caller's: the chunk table
// and the cumsum (ws.cs, ws.delta); then, once ws.states holds each chunk's own state,
// the state pass
cudaError_t simt_cumsum(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                        cudaStream_t stream);
cudaError_t simt_state_pass(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                            cudaStream_t stream);

constexpr int kBwdQ = 64;  // chunk length of the backward kernels

struct GradArgs {
  const void* dy;        // [T, H, P], out dtype
  const float* dfinal;   // [ndocs, H, N, P] or null (zero)
  float* dx;             // [T, H, P]
  float* ddt;            // [T, H]
  float* dA;             // [H]
  float* dB;             // [T, G, N]
  float* dC;             // [T, G, N]
  float* dD;             // [H] or null
  float* ddt_bias;       // [H] or null
  float* dinit;          // [ndocs, H, N, P] or null
};

// Chunk length of the tensor-core backward (bf16 inputs and outputs, P a multiple of 64 up to 256, N = 64 or
// 128, 16-byte aligned x, dy, B and C); ssd_backward takes it when bwd_tc_eligible.
constexpr int kBwdTcQ = 128;
bool bwd_tc_eligible(const Geom& g, const Args& a, const GradArgs& ga);

// Backward workspace beyond the CUDA-core forward's.
struct BwdWs {
  float* dstates;  // [nchunks, H, N, P]: per-chunk sum, then the cotangent at the chunk's end
  float* final;    // [ndocs, H, N, P]: the forward's final states
};

// per (chunk, head) on the tensor cores (g.Q == kBwdTcQ, g.N == 128): mode 0 writes the
// chunk's own state sum_t B_t^T (exp(cs_last - cs_t) delta_t x_t) into ws.states, mode 1
// the cotangent sum sum_t C_t^T (exp(cs_t) dy_t) into bw.dstates
cudaError_t bwd_states_tc(const Geom& g, const Args& a, const GradArgs& ga, const SimtWorkspace& ws,
                          const BwdWs& bw, int mode, int* status, cudaStream_t stream);

// every per-token gradient of each (chunk, head) on the tensor cores (g.Q == kBwdTcQ)
cudaError_t bwd_chunk_tc(const Geom& g, const Args& a, const GradArgs& ga, const SimtWorkspace& ws,
                         const BwdWs& bw, int* status, cudaStream_t stream);

// g.Q must be kBwdQ, or kBwdTcQ when bwd_tc_eligible.
size_t bwd_workspace_bytes(const Geom& g);
cudaError_t bwd_run(const Geom& g, const Args& a, const GradArgs& ga, void* workspace, int* status,
                    cudaStream_t stream);

}  // namespace ssd
