// ssd_simt.cu -- chunk-parallel SSD forward on CUDA cores, fp32 arithmetic.
//
// The block decomposition of "Transformers are SSMs" (paperlayer.ai summary, §6)
// as four kernels over chunks of Q tokens (chunks never straddle a document):
//   cumsum      delta = softplus(dt + dt_bias), inclusive cumsum of delta*A in
//               the chunk (the 1-semiseparable scalar scan of §3.2.2)
//   chunk_state right factors: S_c = B^T (exp(cs_last - cs) * delta * x), the
//               chunk's final state with no input before it (§6.2)
//   state_pass  scalar scan across chunks: H_{c+1} = exp(cs_last,c) H_c + S_c,
//               from the document's initial state (§6.2, App. B.3.2)
//   chunk_scan  diagonal block ((C B^T) o L) (delta x) with zero initial state
//               (§6.1) + left factors exp(cs) C H_c (§6.2) + D x
// This path serves every shape and dtype (fp32 inputs in particular) and is the
// fallback of the tensor-core path.  Packed documents (cu_seqlens) get a chunk
// table built on the device by the varlen_table kernel.
#include <cuda_runtime.h>

#include "ssd_chunks.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kMaxQ = 256;

// Inclusive block-wide sum scan (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ float block_inclusive_scan(float v, float* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    float s = lane < nw ? warp_sums[lane] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    if (lane < nw) warp_sums[lane] = s;
  }
  __syncthreads();
  if (warp > 0) v += warp_sums[warp - 1];
  return v;
}

__device__ __forceinline__ int block_scan_int(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    if (lane < nw) warp_sums[lane] = s;
  }
  __syncthreads();
  if (warp > 0) v += warp_sums[warp - 1];
  return v;
}

// ---- K0: chunk table of packed documents (one block of 1024 threads) ------------
__global__ void __launch_bounds__(1024) k_varlen_table(Geom g, const int32_t* cu,
                                                       SimtWorkspace ws, int* status) {
  __shared__ int bad;
  __shared__ int carry;
  __shared__ int wsum[32];
  if (threadIdx.x == 0) {
    bad = 0;
    carry = 0;
  }
  __syncthreads();
  for (int d = threadIdx.x; d <= g.ndocs; d += blockDim.x) {
    const int64_t v = cu[d];
    if (d == 0 && v != 0) bad = 1;
    if (d == g.ndocs && v != g.tokens) bad = 1;
    if (d > 0 && v < (int64_t)cu[d - 1]) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      ws.total_chunks[0] = 0;
      ws.total_chunks[1] = 0;
      set_status(status, SSD_ERR_BAD_SEQLENS);
    }
    return;
  }
  for (int base = 0; base < g.ndocs; base += blockDim.x) {
    const int d = base + threadIdx.x;
    const int n = d < g.ndocs ? (int)(((int64_t)cu[d + 1] - cu[d] + g.Q - 1) / g.Q) : 0;
    const int incl = block_scan_int(n, wsum);
    const int c0 = carry;
    if (d < g.ndocs) ws.doc_first[d] = c0 + incl - n;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = c0 + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    ws.doc_first[g.ndocs] = carry;
    ws.total_chunks[0] = carry;
    ws.total_chunks[1] = 1;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < g.ndocs; d += blockDim.x)
    for (int k = ws.doc_first[d]; k < ws.doc_first[d + 1]; ++k) ws.chunk_doc[k] = d;
}

// ---- K1: delta and in-chunk cumsum of delta*A -------------------------------------
__global__ void k_cumsum(Geom g, Args a, SimtWorkspace ws) {
  __shared__ float wsum[32];
  const int64_t k = blockIdx.x;
  const int h = blockIdx.y;
  ChunkInfo ci;
  if (!chunk_info(g, a.cu, ws, k, &ci)) return;
  const int l = threadIdx.x;
  float dl = 0.f, la = 0.f;
  if (l < ci.len) {
    const int64_t t = ci.start + l;
    const float z = load_f(a.dt, t * g.H + h, g.in_bf16) + (a.dt_bias ? a.dt_bias[h] : 0.f);
    dl = softplus_f(z);
    la = dl * a.A[h];
  }
  const float cs = block_inclusive_scan(la, wsum);
  if (l < g.Q) {
    const int64_t o = ((int64_t)h * g.nchunks_max + k) * g.Q + l;
    ws.cs[o] = cs;
    ws.delta[o] = dl;
  }
}

// ---- K2: chunk states S_c[n,p] = sum_l B[l,n] w_l x[l,p] ---------------------------
constexpr int kTS = 64;  // n and p tile of chunk_state
__global__ void __launch_bounds__(256) k_chunk_state(Geom g, Args a, SimtWorkspace ws) {
  __shared__ __align__(16) float Bs[32][68];  // rows padded to 16-byte multiples
  __shared__ __align__(16) float Xs[32][68];
  __shared__ float w[32];
  const int64_t k = blockIdx.x;
  const int h = blockIdx.y;
  const int ntp = (g.P + kTS - 1) / kTS;
  const int n0 = (blockIdx.z / ntp) * kTS, p0 = (blockIdx.z % ntp) * kTS;
  ChunkInfo ci;
  if (!chunk_info(g, a.cu, ws, k, &ci)) return;
  const int grp = h / (g.H / g.G);
  const int64_t cso = ((int64_t)h * g.nchunks_max + k) * g.Q;
  const float cs_last = ws.cs[cso + g.Q - 1];
  const int tn = threadIdx.x >> 4, tp = threadIdx.x & 15;
  float acc[4][4] = {};
  for (int l0 = 0; l0 < ci.len; l0 += 32) {
    if (threadIdx.x < 32) {
      const int l = l0 + threadIdx.x;
      w[threadIdx.x] = l < ci.len ? expf(cs_last - ws.cs[cso + l]) * ws.delta[cso + l] : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * kTS; e += 256) {
      const int r = e / kTS, c = e % kTS, l = l0 + r;
      const int64_t t = ci.start + l;
      Bs[r][c] = (l < ci.len && n0 + c < g.N)
                     ? load_f(a.B, (t * g.G + grp) * g.N + n0 + c, g.in_bf16) : 0.f;
      Xs[r][c] = (l < ci.len && p0 + c < g.P)
                     ? w[r] * load_f(a.x, (t * g.H + h) * g.P + p0 + c, g.in_bf16) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 32; ++r) {
      const float4 av = *reinterpret_cast<const float4*>(&Bs[r][tn * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Xs[r][tp * 4]);
      const float a4[4] = {av.x, av.y, av.z, av.w}, b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int64_t so = (k * g.H + h) * (int64_t)g.N * g.P;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + i, p = p0 + tp * 4 + j;
      if (n < g.N && p < g.P) ws.states[so + (int64_t)n * g.P + p] = acc[i][j];
    }
}

// ---- K3: scalar scan of states across the chunks of each document ----------------
__global__ void __launch_bounds__(256) k_state_pass(Geom g, Args a, SimtWorkspace ws) {
  const int d = blockIdx.x, h = blockIdx.y;
  const int64_t NP = (int64_t)g.N * g.P;
  const int64_t e = (int64_t)blockIdx.z * 256 + threadIdx.x;
  if (e >= NP) return;
  int64_t first, cnt;
  if (g.varlen) {
    if (!ws.total_chunks[1]) return;
    first = ws.doc_first[d];
    cnt = ws.doc_first[d + 1] - first;
  } else {
    cnt = (g.seqlen + g.Q - 1) / g.Q;
    first = (int64_t)d * cnt;
  }
  const int64_t so = ((int64_t)d * g.H + h) * NP + e;
  float hc = a.init ? a.init[so] : 0.f;
  // eight chunks per round: their loads are all issued before the dependent updates
  constexpr int kU = 8;
  int64_t c = 0;
  for (; c + kU <= cnt; c += kU) {
    float s[kU], dec[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t kk = first + c + u;
      s[u] = ws.states[(kk * g.H + h) * NP + e];
      dec[u] = ws.cs[((int64_t)h * g.nchunks_max + kk) * g.Q + g.Q - 1];
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      ws.states[((first + c + u) * g.H + h) * NP + e] = hc;
      hc = expf(dec[u]) * hc + s[u];
    }
  }
  for (; c < cnt; ++c) {
    const int64_t kk = first + c;
    const int64_t idx = (kk * g.H + h) * NP + e;
    const float s = ws.states[idx];
    ws.states[idx] = hc;
    hc = expf(ws.cs[((int64_t)h * g.nchunks_max + kk) * g.Q + g.Q - 1]) * hc + s;
  }
  if (a.final_states) a.final_states[so] = hc;
}

// ---- K4: outputs of a chunk --------------------------------------------------------
constexpr int kSL = 32;  // rows (tokens) per block
constexpr int kSP = 64;  // head-dim columns per block
__global__ void __launch_bounds__(256) k_chunk_scan(Geom g, Args a, SimtWorkspace ws) {
  extern __shared__ float sm[];
  const int N = g.N, NS = g.N + 1;      // padded row stride: conflict-free columns
  float* Cs = sm;                        // [kSL][NS]
  float* Bs = Cs + kSL * NS;             // [32][NS]
  float* Xs = Bs + 32 * NS;              // [32][kSP]
  float* Ms = Xs + 32 * kSP;             // [kSL][33]
  float* Hs = Ms + kSL * 33;             // [32][kSP]
  float* csl = Hs + 32 * kSP;            // [kSL]
  float* css = csl + kSL;                // [32]
  float* dls = css + 32;                 // [32]

  const int64_t k = blockIdx.x;
  const int h = blockIdx.y;
  const int ntp = (g.P + kSP - 1) / kSP;
  const int l0 = (blockIdx.z / ntp) * kSL, p0 = (blockIdx.z % ntp) * kSP;
  ChunkInfo ci;
  if (!chunk_info(g, a.cu, ws, k, &ci)) return;
  if (l0 >= ci.len) return;
  const int grp = h / (g.H / g.G);
  const int64_t cso = ((int64_t)h * g.nchunks_max + k) * g.Q;
  const int r2 = (threadIdx.x >> 4) * 2, cp = (threadIdx.x & 15) * 4;

  for (int e = threadIdx.x; e < kSL * N; e += 256) {
    const int r = e / N, n = e % N, l = l0 + r;
    Cs[r * NS + n] = l < ci.len ? load_f(a.C, ((ci.start + l) * g.G + grp) * N + n, g.in_bf16) : 0.f;
  }
  if (threadIdx.x < kSL) {
    const int l = l0 + threadIdx.x;
    csl[threadIdx.x] = l < g.Q ? ws.cs[cso + l] : 0.f;
  }
  __syncthreads();

  // left factors: exp(cs_l) * C_l . H_c  (state entering the chunk)
  float off[2][4] = {};
  const int64_t so = (k * g.H + h) * (int64_t)N * g.P;
  for (int nb = 0; nb < N; nb += 32) {
    for (int e = threadIdx.x; e < 32 * kSP; e += 256) {
      const int r = e / kSP, c = e % kSP;
      Hs[e] = (nb + r < N && p0 + c < g.P) ? ws.states[so + (int64_t)(nb + r) * g.P + p0 + c] : 0.f;
    }
    __syncthreads();
    const int nn = min(32, N - nb);
    for (int r = 0; r < nn; ++r) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float c = Cs[(r2 + i) * NS + nb + r];
#pragma unroll
        for (int j = 0; j < 4; ++j) off[i][j] += c * Hs[r * kSP + cp + j];
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float s = expf(csl[r2 + i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) off[i][j] *= s;
  }

  // diagonal block: sum_{s<=l} (C_l . B_s) exp(cs_l - cs_s) delta_s x_s
  float dia[2][4] = {};
  const int l_hi = min(l0 + kSL, ci.len);  // exclusive
  for (int s0 = 0; s0 < l_hi; s0 += 32) {
    for (int e = threadIdx.x; e < 32 * N; e += 256) {
      const int r = e / N, n = e % N, s = s0 + r;
      Bs[r * NS + n] = s < ci.len ? load_f(a.B, ((ci.start + s) * g.G + grp) * N + n, g.in_bf16) : 0.f;
    }
    for (int e = threadIdx.x; e < 32 * kSP; e += 256) {
      const int r = e / kSP, c = e % kSP, s = s0 + r;
      Xs[e] = (s < ci.len && p0 + c < g.P)
                  ? load_f(a.x, ((ci.start + s) * g.H + h) * g.P + p0 + c, g.in_bf16) : 0.f;
    }
    if (threadIdx.x < 32) {
      const int s = s0 + threadIdx.x;
      css[threadIdx.x] = s < g.Q ? ws.cs[cso + s] : 0.f;
      dls[threadIdx.x] = s < ci.len ? ws.delta[cso + s] : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kSL * 32; e += 256) {
      const int rl = e >> 5, sc = e & 31;
      const int l = l0 + rl, s = s0 + sc;
      float v = 0.f;
      if (s <= l && s < ci.len && l < ci.len) {
        float cb = 0.f;
        for (int n = 0; n < N; ++n) cb += Cs[rl * NS + n] * Bs[sc * NS + n];
        v = cb * expf(csl[rl] - css[sc]) * dls[sc];
      }
      Ms[rl * 33 + sc] = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int sc = 0; sc < 32; ++sc) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float m = Ms[(r2 + i) * 33 + sc];
#pragma unroll
        for (int j = 0; j < 4; ++j) dia[i][j] += m * Xs[sc * kSP + cp + j];
      }
    }
    __syncthreads();
  }

  const float Dh = a.D ? a.D[h] : 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int l = l0 + r2 + i;
    if (l >= ci.len) continue;
    const int64_t row = ((ci.start + l) * g.H + h) * g.P;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = p0 + cp + j;
      if (p >= g.P) continue;
      const float xv = load_f(a.x, row + p, g.in_bf16);
      store_f(a.y, row + p, off[i][j] + dia[i][j] + Dh * xv, g.out_bf16);
    }
  }
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

size_t simt_workspace_bytes(const Geom& g) {
  const size_t nch = (size_t)g.nchunks_max;
  size_t b = 0;
  b += align256(sizeof(float) * (size_t)g.H * nch * g.Q);            // cs
  b += align256(sizeof(float) * (size_t)g.H * nch * g.Q);            // delta
  b += align256(sizeof(float) * nch * g.H * (size_t)g.N * g.P);      // states
  b += align256(sizeof(int) * nch);                                   // chunk_doc
  b += align256(sizeof(int) * ((size_t)g.ndocs + 1));                 // doc_first
  b += align256(sizeof(int) * 2);                                     // total_chunks, ok
  return b;
}

void simt_carve_workspace(const Geom& g, void* base, SimtWorkspace* ws) {
  const size_t nch = (size_t)g.nchunks_max;
  char* p = static_cast<char*>(base);
  ws->cs = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * (size_t)g.H * nch * g.Q);
  ws->delta = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * (size_t)g.H * nch * g.Q);
  ws->states = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * nch * g.H * (size_t)g.N * g.P);
  ws->chunk_doc = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * nch);
  ws->doc_first = reinterpret_cast<int*>(p);
  p += align256(sizeof(int) * ((size_t)g.ndocs + 1));
  ws->total_chunks = reinterpret_cast<int*>(p);
}

int simt_kernels(const Geom& g) {
  int n = g.varlen ? 1 : 0;
  if (g.nchunks_max > 0 && g.H > 0) n += 2;
  if (g.ndocs > 0) n += 1;
  if (g.nchunks_max > 0) n += 1;
  return n;
}

// stage = 0: everything; 1: up to the cumsum (the caller fills the chunk states);
// 2: the state pass only
cudaError_t simt_run(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                     cudaStream_t stream, bool outputs, int stage = 0) {
  if (g.Q < 1 || g.Q > kMaxQ) return cudaErrorInvalidValue;
  if (stage != 2) {
    if (g.varlen) {
      k_varlen_table<<<1, 1024, 0, stream>>>(g, a.cu, ws, status);
    }
    if (g.nchunks_max > 0 && g.H > 0) {
      const int qthreads = ((g.Q + 31) / 32) * 32;
      k_cumsum<<<dim3((unsigned)g.nchunks_max, g.H), qthreads, 0, stream>>>(g, a, ws);
      if (stage == 1) return cudaGetLastError();
      const int tiles_s = ((g.N + kTS - 1) / kTS) * ((g.P + kTS - 1) / kTS);
      k_chunk_state<<<dim3((unsigned)g.nchunks_max, g.H, tiles_s), 256, 0, stream>>>(g, a, ws);
    }
    if (stage == 1) return cudaGetLastError();
  }
  const int64_t NP = (int64_t)g.N * g.P;
  if (g.ndocs > 0) {
    k_state_pass<<<dim3(g.ndocs, g.H, (unsigned)((NP + 255) / 256)), 256, 0, stream>>>(g, a, ws);
  }
  if (stage == 2) return cudaGetLastError();
  if (outputs && g.nchunks_max > 0) {
    const size_t smem =
        sizeof(float) * ((size_t)kSL * (g.N + 1) + 32 * (g.N + 1) + 32 * kSP + kSL * 33 + 32 * kSP +
                         kSL + 64);
    cudaError_t e = cudaFuncSetAttribute(k_chunk_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles_y = ((g.Q + kSL - 1) / kSL) * ((g.P + kSP - 1) / kSP);
    k_chunk_scan<<<dim3((unsigned)g.nchunks_max, g.H, tiles_y), 256, smem, stream>>>(g, a, ws);
  }
  return cudaGetLastError();
}

cudaError_t simt_forward(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                         cudaStream_t stream) {
  return simt_run(g, a, ws, status, stream, true);
}

cudaError_t simt_states(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                        cudaStream_t stream) {
  return simt_run(g, a, ws, status, stream, false);
}

cudaError_t simt_cumsum(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                        cudaStream_t stream) {
  return simt_run(g, a, ws, status, stream, false, 1);
}

cudaError_t simt_state_pass(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                            cudaStream_t stream) {
  return simt_run(g, a, ws, status, stream, false, 2);
}

cudaError_t simt_varlen_table(const Geom& g, const int32_t* cu, const SimtWorkspace& ws, int* status,
                              cudaStream_t stream) {
  k_varlen_table<<<1, 1024, 0, stream>>>(g, cu, ws, status);
  return cudaGetLastError();
}

}  // namespace ssd
