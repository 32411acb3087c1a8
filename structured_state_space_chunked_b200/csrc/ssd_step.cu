// ssd_step.cu -- one token of the recurrence for every sequence of a decode batch.
//
// The recurrent (linear) mode of the selective SSM ("Transformers are SSMs",
// paperlayer.ai summary, §3.4.1; scalar-times-identity A, §2.4), for generation
// one token at a time from a carried state:
//
//   delta = softplus(dt + dt_bias[h]);  S <- exp(delta A[h]) S + delta B^T x;  y = C S + D x
//
// S is the fp32 N x P state of a (sequence, head), read and written in place.  The
// step does 4NP flops per (sequence, head) and moves 8NP state bytes, so it is
// bound by HBM bandwidth: one CTA per (sequence, head) streams its state rows with
// 16-byte loads and stores, the P columns spread over the threads of a row group
// and the rows over the row groups; the C S reduction over rows goes through
// shared memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kStepThreads = 256;

struct StepParams {
  int H, P, N, G;
  int in_bf16, out_bf16;
  const void* x;
  const void* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  const float* dt_bias;
  float* state;
  void* y;
};

__global__ void __launch_bounds__(kStepThreads) ssd_step_kernel(const StepParams p) {
  extern __shared__ float4 red4[];  // [rows in parallel][P / 4]
  float* red = reinterpret_cast<float*>(red4);
  const int bh = blockIdx.x;
  const int b = bh / p.H, h = bh % p.H;
  const int g = h / (p.H / p.G);
  const int c4n = p.P / 4;                 // float4 columns per state row
  const int rpar = kStepThreads / c4n;     // state rows handled in parallel
  const int c4 = threadIdx.x % c4n, r0 = threadIdx.x / c4n;
  const bool active = r0 < rpar;

  const float z = load_f(p.dt, (int64_t)bh, p.in_bf16) + (p.dt_bias ? p.dt_bias[h] : 0.f);
  const float delta = softplus_f(z);
  const float decay = expf(delta * p.A[h]);

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 xv = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
    const int64_t xo = (int64_t)bh * p.P + 4 * c4;
    xv = make_float4(load_f(p.x, xo, p.in_bf16), load_f(p.x, xo + 1, p.in_bf16),
                     load_f(p.x, xo + 2, p.in_bf16), load_f(p.x, xo + 3, p.in_bf16));
    const int64_t bco = ((int64_t)b * p.G + g) * p.N;
    float4* srow = reinterpret_cast<float4*>(p.state + (int64_t)bh * p.N * p.P) + c4;
    for (int n = r0; n < p.N; n += rpar) {
      const float bn = delta * load_f(p.B, bco + n, p.in_bf16);
      const float cn = load_f(p.C, bco + n, p.in_bf16);
      float4 s = srow[(int64_t)n * c4n];
      s.x = fmaf(decay, s.x, bn * xv.x);
      s.y = fmaf(decay, s.y, bn * xv.y);
      s.z = fmaf(decay, s.z, bn * xv.z);
      s.w = fmaf(decay, s.w, bn * xv.w);
      srow[(int64_t)n * c4n] = s;
      acc.x = fmaf(cn, s.x, acc.x);
      acc.y = fmaf(cn, s.y, acc.y);
      acc.z = fmaf(cn, s.z, acc.z);
      acc.w = fmaf(cn, s.w, acc.w);
    }
    reinterpret_cast<float4*>(red + r0 * p.P)[c4] = acc;
  }
  __syncthreads();
  // y[p] = sum over row groups of C S, plus D x
  for (int col = threadIdx.x; col < p.P; col += kStepThreads) {
    float v = 0.f;
    for (int r = 0; r < rpar; ++r) v += red[r * p.P + col];
    const float xc = load_f(p.x, (int64_t)bh * p.P + col, p.in_bf16);
    v = fmaf(p.D ? p.D[h] : 0.f, xc, v);
    store_f(p.y, (int64_t)bh * p.P + col, v, p.out_bf16);
  }
}

bool aligned(const void* q, size_t a) { return ((uintptr_t)q % a) == 0; }

}  // namespace
}  // namespace ssd

extern "C" SSD_API int ssd_step(const ssd_desc_t* desc, const void* x, const void* dt,
                                const float* A, const void* B, const void* C, const float* D,
                                const float* dt_bias, float* state, void* y, ssd_stream_t stream) {
  ssd::NvtxRange nvtx_range("ssd_step");
  using ssd::aligned;
  if (!desc) return SSD_ERR_INVALID_ARG;
  const ssd_desc_t& d = *desc;
  if (d.batch < 0 || d.seqlen != 1 || d.max_docs != 0) return SSD_ERR_INVALID_ARG;
  if (d.nheads < 1 || d.headdim < 1 || d.dstate < 1 || d.ngroups < 1 || d.nheads % d.ngroups)
    return SSD_ERR_INVALID_ARG;
  if ((d.in_dtype != SSD_F32 && d.in_dtype != SSD_BF16) ||
      (d.out_dtype != SSD_F32 && d.out_dtype != SSD_BF16))
    return SSD_ERR_INVALID_ARG;
  if (d.headdim % 4 != 0 || d.headdim / 4 > ssd::kStepThreads) return SSD_ERR_UNSUPPORTED;
  if (d.batch == 0) return SSD_OK;
  if (!x || !dt || !A || !B || !C || !state || !y) return SSD_ERR_INVALID_ARG;
  const size_t ein = d.in_dtype == SSD_BF16 ? 2 : 4, eout = d.out_dtype == SSD_BF16 ? 2 : 4;
  if (!aligned(state, 16) || !aligned(x, ein) || !aligned(dt, ein) || !aligned(B, ein) ||
      !aligned(C, ein) || !aligned(y, eout) || !aligned(A, 4) || !aligned(D, 4) ||
      !aligned(dt_bias, 4))
    return SSD_ERR_INVALID_ARG;
  if (d.batch * d.nheads > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
  ssd::StepParams p;
  p.H = d.nheads;
  p.P = d.headdim;
  p.N = d.dstate;
  p.G = d.ngroups;
  p.in_bf16 = d.in_dtype == SSD_BF16;
  p.out_bf16 = d.out_dtype == SSD_BF16;
  p.x = x;
  p.dt = dt;
  p.A = A;
  p.B = B;
  p.C = C;
  p.D = D;
  p.dt_bias = dt_bias;
  p.state = state;
  p.y = y;
  const int rpar = ssd::kStepThreads / (d.headdim / 4);
  const size_t smem = sizeof(float) * (size_t)rpar * d.headdim;
  if (smem > 48 * 1024) return SSD_ERR_UNSUPPORTED;
  ssd::ssd_step_kernel<<<(unsigned)(d.batch * d.nheads), ssd::kStepThreads, smem,
                         reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
