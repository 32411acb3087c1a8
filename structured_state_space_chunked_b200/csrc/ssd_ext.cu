// ssd_ext.cu -- kernel feature maps on B and C, and denominator normalisation.
//
// "Transformers are SSMs" (paperlayer.ai summary, §7.3) extends SSD the way linear
// attention is extended: a kernel feature map phi on the keys and queries (B and C
// in SSD; SiLU by default) and an optional normalisation by a denominator, which is
// the same scan run on a column of ones in place of X (so phi must be positive for
// the denominator to be).  The ablations (§9.4.3, App. D.4) also try the Based map
// (the second-order Taylor expansion of exp: phi(x) = [1, x, x (x) x / sqrt 2], so
// <phi(a), phi(b)> = 1 + <a,b> + <a,b>^2 / 2) and the ReBased map (x (x) x, so
// <phi(a), phi(b)> = <a,b>^2).  These kernels apply phi elementwise per row and
// divide the numerator by the denominator.  The numerator is ssd_forward's scan; the
// denominator, a scan with a single column, has a warp-per-sequence kernel of its own.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_chunks.cuh"
#include "ssd_ext.h"

namespace ssd {
namespace {

__global__ void fmap_kernel(int kind, int64_t rows, int N, int Nout, int bf16, const void* src,
                            void* dst) {
  const int64_t total = rows * Nout;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / Nout;
    const int j = (int)(i % Nout);
    const int64_t base = r * N;
    float v;
    if (kind == SSD_FMAP_SILU) {
      const float u = load_f(src, base + j, bf16);
      v = u / (1.f + expf(-u));
    } else if (kind == SSD_FMAP_RELU) {
      v = fmaxf(load_f(src, base + j, bf16), 0.f);
    } else if (kind == SSD_FMAP_BASED) {
      if (j == 0) {
        v = 1.f;
      } else if (j <= N) {
        v = load_f(src, base + j - 1, bf16);
      } else {
        const int q = j - 1 - N;
        v = load_f(src, base + q / N, bf16) * load_f(src, base + q % N, bf16) * 0.70710678118654752f;
      }
    } else if (kind == SSD_FMAP_REBASED) {
      v = load_f(src, base + j / N, bf16) * load_f(src, base + j % N, bf16);
    } else {
      v = load_f(src, base + j, bf16);
    }
    store_f(dst, i, v, bf16);
  }
}

// 8 consecutive columns per thread (P a multiple of 8), one division per (token, head)
__global__ void normalize_kernel(int64_t T, int H, int P, int out_bf16, int in_bf16, void* y,
                                 const float* den, const void* x, const float* D) {
  const int64_t total = T * H * (P / 8);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t th = i / (P / 8);
    const int h = (int)(th % H);
    const int64_t e0 = i * 8;
    const float r = 1.f / den[th];
    const float dh = D ? D[h] : 0.f;
    float v[8], xv[8];
    if (out_bf16) {
      const uint4 q = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(y) + e0);
      const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(q2[k]);
        v[2 * k] = f.x;
        v[2 * k + 1] = f.y;
      }
    } else {
      const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(y) + e0);
      const float4 a = q[0], b = q[1];
      v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    }
    if (D) {
#pragma unroll
      for (int k = 0; k < 8; ++k) xv[k] = load_f(x, e0 + k, in_bf16);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) xv[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = fmaf(dh, xv[k], v[k] * r);
    if (out_bf16) {
      uint4 q;
      __nv_bfloat162* q2 = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
      for (int k = 0; k < 4; ++k) q2[k] = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(y) + e0) = q;
    } else {
      float4* q = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + e0);
      q[0] = make_float4(v[0], v[1], v[2], v[3]);
      q[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

__global__ void normalize_scalar_kernel(int64_t T, int H, int P, int out_bf16, int in_bf16, void* y,
                                        const float* den, const void* x, const float* D) {
  const int64_t total = T * H * P;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t th = i / P;
    const int h = (int)(th % H);
    float v = load_f(y, i, out_bf16) / den[th];
    if (D) v = fmaf(D[h], load_f(x, i, in_bf16), v);
    store_f(y, i, v, out_bf16);
  }
}

// The denominator: the scan on a ones column, den_t = <C_t, z_t> with
// z_t = exp(delta_t A) z_{t-1} + delta_t B_t (an N-vector per document and head, zero
// at each document's start).  In chunks of 64 tokens, as the block decomposition of
// §6 runs the scan: (1) each chunk runs the recurrence from zero and keeps its end
// state and log decay; (2) a scan over the chunks of each document turns those into
// the state entering every chunk; (3) each chunk runs the recurrence again from its
// entering state and writes den.  Steps 1 and 3 give one warp to a (chunk, head);
// lane l holds state elements l, l + 32, ...; the per-token dot products of step 3
// are summed 32 tokens at a time through shared memory.
constexpr int kDenWarps = 4;
template <int E, bool OUT>
__global__ void __launch_bounds__(32 * kDenWarps)
    den_chunk_kernel(Geom g, const int32_t* cu, SimtWorkspace ws, const void* dt, const float* A,
                     const float* dt_bias, const void* B, const void* C, float* den) {
  __shared__ float part[kDenWarps][32][33];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kDenWarps + w;  // (chunk, head), heads fastest
  if (item >= g.nchunks_max * g.H) return;
  const int64_t k = item / g.H;
  const int h = (int)(item % g.H), grp = h / (g.H / g.G), N = g.N;
  ChunkInfo ci;
  if (!chunk_info(g, cu, ws, k, &ci)) return;
  const float a_h = A[h], bias = dt_bias ? dt_bias[h] : 0.f;
  float* zs = ws.states + (k * g.H + h) * (int64_t)N;
  float z[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int n = lane + 32 * e;
    z[e] = (OUT && n < N) ? zs[n] : 0.f;
  }
  float cs = 0.f;
  for (int tb = 0; tb < ci.len; tb += 32) {
    const int nt = min(32, ci.len - tb);
#pragma unroll 4
    for (int u = 0; u < nt; ++u) {
      const int64_t t = ci.start + tb + u;
      const float delta = softplus_f(load_f(dt, t * g.H + h, g.in_bf16) + bias);
      const float decay = expf(delta * a_h);
      cs = fmaf(delta, a_h, cs);
      const int64_t row = (t * g.G + grp) * (int64_t)N;
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int n = lane + 32 * e;
        if (n < N) {
          z[e] = fmaf(decay, z[e], delta * load_f(B, row + n, g.in_bf16));
          if (OUT) sdot = fmaf(load_f(C, row + n, g.in_bf16), z[e], sdot);
        }
      }
      if (OUT) part[w][u][lane] = sdot;
    }
    if (OUT) {
      __syncwarp();
      if (lane < nt) {
        float tot = 0.f;
#pragma unroll 8
        for (int q = 0; q < 32; ++q) tot += part[w][lane][q];
        den[(ci.start + tb + lane) * g.H + h] = tot;
      }
      __syncwarp();
    }
  }
  if (!OUT) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int n = lane + 32 * e;
      if (n < N) zs[n] = z[e];
    }
    if (lane == 0) ws.cs[((int64_t)h * g.nchunks_max + k) * g.Q + g.Q - 1] = cs;
  }
}

// Steps (1) and (3) with the chunk's rows staged in shared memory: one CTA per
// (chunk, block of 8 heads of one B/C group), one warp per head.  The chunk's B and C
// rows (input dtype) and dt of the 8 heads are copied in once by the whole CTA
// (consecutive threads on consecutive elements), so the serial token loop of each
// warp reads shared memory only.  Same arithmetic, in the same order, as
// den_chunk_kernel.
constexpr int kDenHeads = 8;
template <int E, bool OUT, typename TIn>
__global__ void __launch_bounds__(32 * kDenHeads)
    den_chunk_staged_kernel(Geom g, const int32_t* cu, SimtWorkspace ws, const void* dt,
                            const float* A, const float* dt_bias, const void* B, const void* C,
                            float* den) {
  extern __shared__ __align__(16) unsigned char den_smem[];
  TIn* sB = reinterpret_cast<TIn*>(den_smem);                 // [Q][N]
  TIn* sC = sB + (size_t)kDenQ * g.N;                          // [Q][N]
  float* sdt = reinterpret_cast<float*>(sC + (size_t)kDenQ * g.N);  // [Q][kDenHeads]
  float (*part)[33] = reinterpret_cast<float (*)[33]>(sdt + kDenQ * kDenHeads);  // [8 warps * 32][33]
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t k = blockIdx.x;
  const int h0 = blockIdx.y * kDenHeads, h = h0 + w, grp = h0 / (g.H / g.G), N = g.N;
  ChunkInfo ci;
  if (!chunk_info(g, cu, ws, k, &ci)) return;
  // stage the chunk: B and C rows of the group, dt of the 8 heads
  const int64_t row0 = (ci.start * g.G + grp) * (int64_t)N;
  const int64_t rstride = (int64_t)g.G * N;
  for (int i = threadIdx.x; i < ci.len * N; i += blockDim.x) {
    const int t = i / N, n = i % N;
    sB[i] = reinterpret_cast<const TIn*>(B)[row0 + t * rstride + n];
    sC[i] = reinterpret_cast<const TIn*>(C)[row0 + t * rstride + n];
  }
  for (int i = threadIdx.x; i < ci.len * kDenHeads; i += blockDim.x) {
    const int t = i / kDenHeads, hh = i % kDenHeads;
    sdt[i] = load_f(dt, (ci.start + t) * g.H + h0 + hh, g.in_bf16);
  }
  __syncthreads();
  const float a_h = A[h], bias = dt_bias ? dt_bias[h] : 0.f;
  float* zs = ws.states + (k * g.H + h) * (int64_t)N;
  float z[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int n = lane + 32 * e;
    z[e] = (OUT && n < N) ? zs[n] : 0.f;
  }
  float cs = 0.f;
  for (int tb = 0; tb < ci.len; tb += 32) {
    const int nt = min(32, ci.len - tb);
    for (int u = 0; u < nt; ++u) {
      const int t = tb + u;
      const float delta = softplus_f(sdt[t * kDenHeads + w] + bias);
      const float decay = expf(delta * a_h);
      cs = fmaf(delta, a_h, cs);
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int n = lane + 32 * e;
        if (n < N) {
          z[e] = fmaf(decay, z[e], delta * (float)sB[t * N + n]);
          if (OUT) sdot = fmaf((float)sC[t * N + n], z[e], sdot);
        }
      }
      if (OUT) part[w * 32 + u][lane] = sdot;
    }
    if (OUT) {
      __syncwarp();
      if (lane < nt) {
        float tot = 0.f;
#pragma unroll 8
        for (int q = 0; q < 32; ++q) tot += part[w * 32 + lane][q];
        den[(ci.start + tb + lane) * g.H + h] = tot;
      }
      __syncwarp();
    }
  }
  if (!OUT) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int n = lane + 32 * e;
      if (n < N) zs[n] = z[e];
    }
    if (lane == 0) ws.cs[((int64_t)h * g.nchunks_max + k) * g.Q + g.Q - 1] = cs;
  }
}

size_t den_staged_smem(const Geom& g) {
  const size_t es = g.in_bf16 ? 2 : 4;
  return 2 * (size_t)kDenQ * g.N * es + sizeof(float) * (kDenQ * kDenHeads + 32 * kDenHeads * 33);
}

// (2): per (document, head, state element), the chunks' end states become entering
// states; eight chunks of loads are issued ahead of their dependent updates
__global__ void __launch_bounds__(256) den_pass_kernel(Geom g, SimtWorkspace ws) {
  const int d = blockIdx.x, h = blockIdx.y;
  const int n = blockIdx.z * 256 + threadIdx.x;
  if (n >= g.N) return;
  if (g.varlen && !ws.total_chunks[1]) return;
  int64_t first;
  const int64_t cnt = doc_chunks(g, ws, d, &first);
  float carry = 0.f;
  constexpr int kU = 8;
  int64_t c = 0;
  for (; c + kU <= cnt; c += kU) {
    float s[kU], ld[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t kk = first + c + u;
      s[u] = ws.states[(kk * g.H + h) * (int64_t)g.N + n];
      ld[u] = ws.cs[((int64_t)h * g.nchunks_max + kk) * g.Q + g.Q - 1];
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      ws.states[((first + c + u) * g.H + h) * (int64_t)g.N + n] = carry;
      carry = fmaf(expf(ld[u]), carry, s[u]);
    }
  }
  for (; c < cnt; ++c) {
    const int64_t kk = first + c;
    const int64_t idx = (kk * g.H + h) * (int64_t)g.N + n;
    const float s = ws.states[idx];
    ws.states[idx] = carry;
    carry = fmaf(expf(ws.cs[((int64_t)h * g.nchunks_max + kk) * g.Q + g.Q - 1]), carry, s);
  }
}

unsigned grid_for(int64_t n) {
  const int64_t b = (n + 255) / 256;
  return (unsigned)(b < 1 ? 1 : b > 148 * 16 ? 148 * 16 : b);
}

}  // namespace

int fmap_dim(int kind, int N) {
  switch (kind) {
    case SSD_FMAP_NONE:
    case SSD_FMAP_SILU:
    case SSD_FMAP_RELU:
      return N;
    case SSD_FMAP_BASED:
      return 1 + N + N * N;
    case SSD_FMAP_REBASED:
      return N * N;
    default:
      return -1;
  }
}

cudaError_t fmap_apply(int kind, int64_t rows, int N, int Nout, int bf16, const void* src, void* dst,
                       cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  fmap_kernel<<<grid_for(rows * Nout), 256, 0, stream>>>(kind, rows, N, Nout, bf16, src, dst);
  return cudaGetLastError();
}

cudaError_t normalize_apply(int64_t T, int H, int P, int out_bf16, int in_bf16, void* y,
                            const float* den, const void* x, const float* D, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  if (P % 8 == 0 && ((uintptr_t)y % 16) == 0)
    normalize_kernel<<<grid_for(T * H * (P / 8)), 256, 0, stream>>>(T, H, P, out_bf16, in_bf16, y, den,
                                                                    x, D);
  else
    normalize_scalar_kernel<<<grid_for(T * H * P), 256, 0, stream>>>(T, H, P, out_bf16, in_bf16, y,
                                                                     den, x, D);
  return cudaGetLastError();
}

bool den_scan_supported(int N) { return N >= 1 && N <= 32 * 32; }

cudaError_t den_scan(const Geom& g, const int32_t* cu, void* workspace, int* status, const void* dt,
                     const float* A, const float* dt_bias, const void* B, const void* C, float* den,
                     cudaStream_t stream) {
  if (g.Q != kDenQ || g.P != 1) return cudaErrorInvalidValue;
  SimtWorkspace ws;
  simt_carve_workspace(g, workspace, &ws);
  if (g.varlen) {
    cudaError_t e = simt_varlen_table(g, cu, ws, status, stream);
    if (e != cudaSuccess) return e;
  }
  const int64_t items = g.nchunks_max * g.H;
  if (items <= 0) return cudaSuccess;
  const size_t sm = den_staged_smem(g);
  if ((g.H / g.G) % kDenHeads == 0 && sm <= 227 * 1024) {
    // chunk rows staged in shared memory (8 heads of a group per CTA)
    const dim3 sgrid((unsigned)g.nchunks_max, (unsigned)(g.H / kDenHeads));
    const int E = (g.N + 31) / 32;
    cudaError_t e = cudaSuccess;
    auto run = [&](auto kern) {
      if (e != cudaSuccess) return;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e == cudaSuccess) {
        kern<<<sgrid, 32 * kDenHeads, sm, stream>>>(g, cu, ws, dt, A, dt_bias, B, C, den);
        e = cudaGetLastError();
      }
    };
#define SSD_DEN_STAGED(EV, OUTV)                                                        \
  (g.in_bf16 ? run(den_chunk_staged_kernel<EV, OUTV, __nv_bfloat16>)                     \
             : run(den_chunk_staged_kernel<EV, OUTV, float>))
#define SSD_DEN_SPICK(OUTV)                                \
  if (E <= 1) SSD_DEN_STAGED(1, OUTV);                     \
  else if (E <= 2) SSD_DEN_STAGED(2, OUTV);                \
  else if (E <= 4) SSD_DEN_STAGED(4, OUTV);                \
  else if (E <= 8) SSD_DEN_STAGED(8, OUTV);                \
  else if (E <= 16) SSD_DEN_STAGED(16, OUTV);              \
  else SSD_DEN_STAGED(32, OUTV)
    SSD_DEN_SPICK(false);
    if (e == cudaSuccess && g.ndocs > 0) {
      den_pass_kernel<<<dim3(g.ndocs, g.H, (unsigned)((g.N + 255) / 256)), 256, 0, stream>>>(g, ws);
      e = cudaGetLastError();
    }
    SSD_DEN_SPICK(true);
#undef SSD_DEN_SPICK
#undef SSD_DEN_STAGED
    return e;
  }
  const unsigned grid = (unsigned)((items + kDenWarps - 1) / kDenWarps);
  const int E = (g.N + 31) / 32;
#define SSD_DEN_CASE(EV, OUTV)                                                                   \
  den_chunk_kernel<EV, OUTV><<<grid, 32 * kDenWarps, 0, stream>>>(g, cu, ws, dt, A, dt_bias, B, C, \
                                                                  den)
#define SSD_DEN_PICK(OUTV)              \
  if (E <= 1) SSD_DEN_CASE(1, OUTV);    \
  else if (E <= 2) SSD_DEN_CASE(2, OUTV); \
  else if (E <= 4) SSD_DEN_CASE(4, OUTV); \
  else if (E <= 8) SSD_DEN_CASE(8, OUTV); \
  else if (E <= 16) SSD_DEN_CASE(16, OUTV); \
  else SSD_DEN_CASE(32, OUTV)
  SSD_DEN_PICK(false);
  if (g.ndocs > 0)
    den_pass_kernel<<<dim3(g.ndocs, g.H, (unsigned)((g.N + 255) / 256)), 256, 0, stream>>>(g, ws);
  SSD_DEN_PICK(true);
#undef SSD_DEN_PICK
#undef SSD_DEN_CASE
  return cudaGetLastError();
}

}  // namespace ssd
