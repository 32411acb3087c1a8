// ssd_bwd.cu -- backward pass of the chunked SSD scan on CUDA cores, fp32.
//
// The gradient of sum_t <dy_t, y_t> + <dfinal, final_state> with respect to x, dt, A,
// B, C, D, dt_bias and the initial states.  The pages state only the training cost
// of the layer ("Transformers are SSMs", paperlayer.ai summary, §3.4 and §6); this is
// the chain rule applied to the block decomposition of §6, one chunk of Q tokens at a
// time.  Inside a chunk with entering state H_c, in-chunk log decay cs_t (cumsum of
// delta A) and cotangent dE of the state at the chunk's end, the state after token t
// is S_t = exp(cs_t) H_c + sum_{s<=t} exp(cs_t - cs_s) delta_s B_s x_s^T, and
//
//   dC_t   = exp(cs_t) H_c dy_t + sum_{s<=t} exp(cs_t - cs_s) delta_s <x_s, dy_t> B_s
//   gB_s   = sum_{u>=s} exp(cs_u - cs_s) <C_u, B_s> dy_u + exp(cs_last - cs_s) dE^T B_s
//   dx_s   = delta_s gB_s + D dy_s
//   dB_s   = delta_s (sum_{u>=s} exp(cs_u - cs_s) <x_s, dy_u> C_u + exp(cs_last - cs_s) dE x_s)
//   dcs_k  = <C_k, dC_k> - delta_k <x_k, gB_k> + [k last] <dE, S_last>
//   ddelta_k = <x_k, gB_k> + A sum_{t>=k} dcs_t,   dA = sum_k delta_k sum_{t>=k} dcs_t
//   ddt_k  = ddelta_k sigmoid(dt_k + dt_bias),      dD = sum <dy, x>
//
// The cotangents of the chunk boundaries come from a reverse scan over the chunks of
// each document: dH_c = sum_{t in c} exp(cs_t) C_t dy_t^T + exp(cs_last,c) dH_{c+1},
// from dH = dfinal after the last chunk; dH_0 is the initial-state gradient.
//
// Kernels: the CUDA-core forward up to its state pass (cs, delta, entering states,
// final states), then
//   kb_chunk_dstate  sum_t exp(cs_t) C_t dy_t^T per chunk
//   kb_state_pass    the reverse scan above
//   kb_chunk         every per-token gradient of one (chunk, head) from 64 x 64 tiles
//                    in shared memory; dB and dC add over the heads of a group
//                    (fp32 atomics), dA, dD and ddt_bias over chunks.
// For bf16 inputs with P a multiple of 64 (up to 256) and N = 64 or 128 (bwd_tc_eligible) the chunks are 128
// tokens long and ssd_bwd_tc.cu takes over the products: kb_chunk_tc in place of
// kb_chunk and, for N = 128, kb_states_tc in place of the two chunk-state products.
#include <cuda_runtime.h>

#include "ssd_bwd.h"
#include "ssd_chunks.cuh"

namespace ssd {
namespace {

constexpr int kLD = 68;            // row stride of the 64 x 64 shared tiles (16-byte rows)
constexpr int kTileF = 64 * kLD;   // floats per tile

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// up to six arrays zeroed by one launch: array k takes blocks first[k] .. first[k+1] - 1,
// each block a run of kZeroRun consecutive elements
constexpr int kZeroRun = 256 * 8;
struct ZeroList {
  float* p[6];
  int64_t n[6];
  int64_t first[7];
  int count;
};
__global__ void __launch_bounds__(256) kb_zero(ZeroList z) {
  for (int64_t blk = blockIdx.x; blk < z.first[z.count]; blk += gridDim.x) {
    int k = 0;
    while (blk >= z.first[k + 1]) ++k;
    const int64_t base = (blk - z.first[k]) * kZeroRun;
    float* q = z.p[k];
#pragma unroll
    for (int u = 0; u < kZeroRun / 256; ++u) {
      const int64_t i = base + u * 256 + threadIdx.x;
      if (i < z.n[k]) q[i] = 0.f;
    }
  }
}

// dS_c[n][p] = sum_l exp(cs_l) C[l][n] dy[l][p] over the tokens of chunk c
__global__ void __launch_bounds__(256) kb_chunk_dstate(Geom g, Args a, GradArgs ga, SimtWorkspace ws,
                                                       BwdWs bw) {
  __shared__ __align__(16) float Cs[32][68];  // rows padded to 16-byte multiples
  __shared__ __align__(16) float Ys[32][68];
  __shared__ float w[32];
  const int64_t k = blockIdx.x;
  const int h = blockIdx.y;
  const int ntp = (g.P + 63) / 64;
  const int n0 = (blockIdx.z / ntp) * 64, p0 = (blockIdx.z % ntp) * 64;
  ChunkInfo ci;
  if (!chunk_info(g, a.cu, ws, k, &ci)) return;
  const int grp = h / (g.H / g.G);
  const int64_t cso = ((int64_t)h * g.nchunks_max + k) * g.Q;
  const int tn = threadIdx.x >> 4, tp = threadIdx.x & 15;
  float acc[4][4] = {};
  for (int l0 = 0; l0 < ci.len; l0 += 32) {
    if (threadIdx.x < 32) {
      const int l = l0 + threadIdx.x;
      w[threadIdx.x] = l < ci.len ? expf(ws.cs[cso + l]) : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * 64; e += 256) {
      const int r = e / 64, c = e % 64, l = l0 + r;
      const int64_t t = ci.start + l;
      Cs[r][c] = (l < ci.len && n0 + c < g.N) ? load_f(a.C, (t * g.G + grp) * g.N + n0 + c, g.in_bf16)
                                              : 0.f;
      Ys[r][c] = (l < ci.len && p0 + c < g.P)
                     ? w[r] * load_f(ga.dy, (t * g.H + h) * g.P + p0 + c, g.out_bf16)
                     : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 32; ++r) {
      const float4 av = *reinterpret_cast<const float4*>(&Cs[r][tn * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Ys[r][tp * 4]);
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
      if (n < g.N && p < g.P) bw.dstates[so + (int64_t)n * g.P + p] = acc[i][j];
    }
}

// Reverse scan over the chunks of each document, one state element per thread:
// dstates[c] becomes the cotangent of the state at the end of chunk c.
__global__ void __launch_bounds__(256) kb_state_pass(Geom g, Args a, GradArgs ga, SimtWorkspace ws,
                                                     BwdWs bw) {
  const int d = blockIdx.x, h = blockIdx.y;
  const int64_t NP = (int64_t)g.N * g.P;
  const int64_t e = (int64_t)blockIdx.z * 256 + threadIdx.x;
  if (e >= NP) return;
  if (g.varlen && !ws.total_chunks[1]) return;
  int64_t first;
  const int64_t cnt = doc_chunks(g, ws, d, &first);
  const int64_t so = ((int64_t)d * g.H + h) * NP + e;
  float carry = ga.dfinal ? ga.dfinal[so] : 0.f;
  // eight chunks per round: their loads are all issued before the dependent updates
  constexpr int kU = 8;
  int64_t c = cnt - 1;
  for (; c + 1 >= kU; c -= kU) {
    float s[kU], dec[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t kk = first + c - u;
      s[u] = bw.dstates[(kk * g.H + h) * NP + e];
      dec[u] = ws.cs[((int64_t)h * g.nchunks_max + kk) * g.Q + g.Q - 1];
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      bw.dstates[((first + c - u) * g.H + h) * NP + e] = carry;
      carry = fmaf(expf(dec[u]), carry, s[u]);
    }
  }
  for (; c >= 0; --c) {
    const int64_t kk = first + c;
    const int64_t idx = (kk * g.H + h) * NP + e;
    const float s = bw.dstates[idx];
    bw.dstates[idx] = carry;
    carry = fmaf(expf(ws.cs[((int64_t)h * g.nchunks_max + kk) * g.Q + g.Q - 1]), carry, s);
  }
  if (ga.dinit) ga.dinit[so] = carry;
  (void)a;
}

// acc[i][j] += sum_{k<64} A(m, k) B(k, n) with m = 4 ty + i, n = 4 tx + j, B stored
// [k][n].  mac_nn: A stored [m][k]; mac_tn: A stored [k][m].  All shared-memory reads
// are 16-byte vectors.
__device__ __forceinline__ float pick(const float4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

__device__ __forceinline__ void fma_row(float (&r)[4], float a, const float4& b) {
  r[0] = fmaf(a, b.x, r[0]);
  r[1] = fmaf(a, b.y, r[1]);
  r[2] = fmaf(a, b.z, r[2]);
  r[3] = fmaf(a, b.w, r[3]);
}

__device__ __forceinline__ void mac_nn(float (&acc)[4][4], const float* A, const float* B, int ty,
                                       int tx) {
#pragma unroll 2
  for (int k0 = 0; k0 < 64; k0 += 4) {
    float4 a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(A + (4 * ty + i) * kLD + k0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 b = *reinterpret_cast<const float4*>(B + (k0 + q) * kLD + 4 * tx);
#pragma unroll
      for (int i = 0; i < 4; ++i) fma_row(acc[i], pick(a[i], q), b);
    }
  }
}

__device__ __forceinline__ void mac_tn(float (&acc)[4][4], const float* A, const float* B, int ty,
                                       int tx) {
#pragma unroll 4
  for (int k = 0; k < 64; ++k) {
    const float4 a = *reinterpret_cast<const float4*>(A + k * kLD + 4 * ty);
    const float4 b = *reinterpret_cast<const float4*>(B + k * kLD + 4 * tx);
    fma_row(acc[0], a.x, b);
    fma_row(acc[1], a.y, b);
    fma_row(acc[2], a.z, b);
    fma_row(acc[3], a.w, b);
  }
}

// T[r][c] = f(r, c), and its transpose T[c][r] = f(r, c), for r, c < 64 (c is the
// contiguous index of the source, so the global reads coalesce either way)
template <class F>
__device__ __forceinline__ void fill(float* T, F f) {
  for (int e = threadIdx.x; e < 64 * 64; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    T[r * kLD + c] = f(r, c);
  }
}
template <class F>
__device__ __forceinline__ void fill_t(float* T, F f) {
  for (int e = threadIdx.x; e < 64 * 64; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    T[c * kLD + r] = f(r, c);
  }
}

// sum over the 16 threads that share ty (16 consecutive lanes)
__device__ __forceinline__ float row_sum16(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// block-wide sum (256 threads), returned to every thread
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += red[w];
  return s;
}

// Every per-token gradient of one (chunk, head); 256 threads, kBwdQ = 64 tokens.
__global__ void __launch_bounds__(256) kb_chunk(Geom g, Args a, GradArgs ga, SimtWorkspace ws,
                                                BwdWs bw) {
  extern __shared__ float sm[];
  float* W = sm;              // W[t][s] = exp(cs_t - cs_s) <x_s, dy_t>, s <= t
  float* V = W + kTileF;      // V[u][s] = exp(cs_u - cs_s) <C_u, B_s>, s <= u
  float* TA = V + kTileF;     // operand tiles
  float* TB = TA + kTileF;
  float* TC = TB + kTileF;
  float* TD = TC + kTileF;
  float* vcs = TD + kTileF;   // cs_t
  float* vdl = vcs + 64;      // delta_t
  float* vecs = vdl + 64;     // exp(cs_t)
  float* veq = vecs + 64;     // exp(cs_last - cs_t)
  float* vdcs = veq + 64;     // <C_t, dC_t>, then the reverse cumsum of dcs
  float* vxg = vdcs + 64;     // <x_t, gB_t>
  float* red = vxg + 64;      // [8]

  const int64_t k = blockIdx.x;
  const int h = blockIdx.y;
  ChunkInfo ci;
  if (!chunk_info(g, a.cu, ws, k, &ci)) return;
  const int len = ci.len, tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int N = g.N, P = g.P, H = g.H, G = g.G, grp = h / (H / G);
  const int64_t NP = (int64_t)N * P, t0 = ci.start;
  const int64_t cso = ((int64_t)h * g.nchunks_max + k) * g.Q;
  const float cs_last = ws.cs[cso + g.Q - 1];
  if (tid < 64) {
    const float c = ws.cs[cso + tid];
    vcs[tid] = c;
    vdl[tid] = ws.delta[cso + tid];
    vecs[tid] = expf(c);
    veq[tid] = expf(cs_last - c);
    vdcs[tid] = 0.f;
    vxg[tid] = 0.f;
  }
  __syncthreads();
  const float* Hc = ws.states + (k * H + h) * NP;    // state entering the chunk
  const float* dE = bw.dstates + (k * H + h) * NP;   // cotangent of the state at its end
  auto xv = [&](int r, int p) -> float {
    return (r < len && p < P) ? load_f(a.x, ((t0 + r) * H + h) * P + p, g.in_bf16) : 0.f;
  };
  auto dyv = [&](int r, int p) -> float {
    return (r < len && p < P) ? load_f(ga.dy, ((t0 + r) * H + h) * P + p, g.out_bf16) : 0.f;
  };
  auto bv = [&](int r, int n) -> float {
    return (r < len && n < N) ? load_f(a.B, ((t0 + r) * G + grp) * N + n, g.in_bf16) : 0.f;
  };
  auto cv = [&](int r, int n) -> float {
    return (r < len && n < N) ? load_f(a.C, ((t0 + r) * G + grp) * N + n, g.in_bf16) : 0.f;
  };
  auto st = [&](const float* S, int n, int p) -> float {
    return (n < N && p < P) ? S[(int64_t)n * P + p] : 0.f;
  };

  // 1. W, and <dy_t, x_t> on its diagonal for dD
  float dDp = 0.f;
  {
    float acc[4][4] = {};
    for (int p0 = 0; p0 < P; p0 += 64) {
      fill(TA, [&](int r, int c) { return xv(r, p0 + c); });
      fill_t(TB, [&](int r, int c) { return dyv(r, p0 + c); });
      __syncthreads();
      mac_nn(acc, TA, TB, ty, tx);  // acc = <x_s, dy_t>, s = 4ty+i, t = 4tx+j
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s = 4 * ty + i, t = 4 * tx + j;
        if (s == t && t < len) dDp += acc[i][j];
        W[t * kLD + s] = (s <= t && t < len) ? expf(vcs[t] - vcs[s]) * acc[i][j] : 0.f;
      }
  }
  // 2. V
  {
    float acc[4][4] = {};
    for (int n0 = 0; n0 < N; n0 += 64) {
      fill(TA, [&](int r, int c) { return cv(r, n0 + c); });
      fill_t(TB, [&](int r, int c) { return bv(r, n0 + c); });
      __syncthreads();
      mac_nn(acc, TA, TB, ty, tx);  // acc = <C_u, B_s>, u = 4ty+i, s = 4tx+j
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int u = 4 * ty + i, s = 4 * tx + j;
        V[u * kLD + s] = (s <= u && u < len) ? expf(vcs[u] - vcs[s]) * acc[i][j] : 0.f;
      }
  }
  __syncthreads();

  // 3. dC and dB, 64 state rows at a time
  for (int n0 = 0; n0 < N; n0 += 64) {
    fill(TB, [&](int r, int c) { return vdl[r] * bv(r, n0 + c); });
    fill(TC, [&](int r, int c) { return cv(r, n0 + c); });
    __syncthreads();
    // the inter-chunk terms go into the same accumulators through row-scaled tiles
    float aC[4][4] = {}, aB[4][4] = {};
    mac_nn(aC, W, TB, ty, tx);  // sum_s W[t][s] delta_s B_s[n]
    mac_tn(aB, W, TC, ty, tx);  // sum_u W[u][s] C_u[n]
    for (int p0 = 0; p0 < P; p0 += 64) {
      __syncthreads();
      fill(TA, [&](int r, int c) { return vecs[r] * dyv(r, p0 + c); });
      fill_t(TD, [&](int r, int c) { return st(Hc, n0 + r, p0 + c); });
      __syncthreads();
      mac_nn(aC, TA, TD, ty, tx);  // + exp(cs_t) sum_p dy_t[p] H_c[n][p]
      __syncthreads();
      fill(TA, [&](int r, int c) { return veq[r] * xv(r, p0 + c); });
      fill_t(TD, [&](int r, int c) { return st(dE, n0 + r, p0 + c); });
      __syncthreads();
      mac_nn(aB, TA, TD, ty, tx);  // + exp(cs_last - cs_s) sum_p x_s[p] dE[n][p]
    }
    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * ty + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + 4 * tx + j;
        const float dc = aC[i][j];
        const float db = vdl[r] * aB[i][j];
        if (r < len && n < N) {
          const int64_t o = ((t0 + r) * G + grp) * N + n;
          atomicAdd(ga.dC + o, dc);
          atomicAdd(ga.dB + o, db);
        }
        part[i] = fmaf(TC[r * kLD + 4 * tx + j], dc, part[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v = row_sum16(part[i]);
      if (tx == 0) vdcs[4 * ty + i] += v;
    }
    __syncthreads();
  }

  // 4. gB, dx and <x, gB>, 64 head-dim columns at a time
  const float Dh = a.D ? a.D[h] : 0.f;
  for (int p0 = 0; p0 < P; p0 += 64) {
    fill(TA, [&](int r, int c) { return dyv(r, p0 + c); });
    fill(TC, [&](int r, int c) { return xv(r, p0 + c); });
    __syncthreads();
    float acc[4][4] = {};
    mac_tn(acc, V, TA, ty, tx);  // sum_u V[u][s] dy_u[p]
    for (int n0 = 0; n0 < N; n0 += 64) {
      __syncthreads();
      fill(TB, [&](int r, int c) { return veq[r] * bv(r, n0 + c); });
      fill(TD, [&](int r, int c) { return st(dE, n0 + r, p0 + c); });
      __syncthreads();
      mac_nn(acc, TB, TD, ty, tx);  // + exp(cs_last - cs_s) sum_n B_s[n] dE[n][p]
    }
    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int s = 4 * ty + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int p = p0 + 4 * tx + j;
        const float gb = acc[i][j];
        if (s < len && p < P)
          ga.dx[((t0 + s) * H + h) * P + p] = fmaf(vdl[s], gb, Dh * TA[s * kLD + 4 * tx + j]);
        part[i] = fmaf(TC[s * kLD + 4 * tx + j], gb, part[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v = row_sum16(part[i]);
      if (tx == 0) vxg[4 * ty + i] += v;
    }
    __syncthreads();
  }

  // 5. <dE, S_last>: S_last enters the next chunk, or is the document's final state
  int64_t first;
  const int64_t cnt = doc_chunks(g, ws, ci.doc, &first);
  const float* Hend = (k == first + cnt - 1) ? bw.final + ((int64_t)ci.doc * H + h) * NP
                                             : ws.states + ((k + 1) * H + h) * NP;
  float sp = 0.f;
  for (int64_t e = tid; e < NP; e += blockDim.x) sp = fmaf(dE[e], Hend[e], sp);
  const float scal = block_sum(sp, red);

  // 6. dcs, its reverse cumsum, ddelta, ddt and the per-head sums
  if (tid == 0) {
    float run = 0.f;
    for (int l = len - 1; l >= 0; --l) {
      run += vdcs[l] - vdl[l] * vxg[l] + (l == len - 1 ? scal : 0.f);
      vdcs[l] = run;
    }
  }
  __syncthreads();
  float pA = 0.f, pb = 0.f;
  if (tid < len) {
    const int64_t t = t0 + tid;
    const float ddelta = fmaf(a.A[h], vdcs[tid], vxg[tid]);
    const float z = load_f(a.dt, t * H + h, g.in_bf16) + (a.dt_bias ? a.dt_bias[h] : 0.f);
    const float gdt = ddelta / (1.f + expf(-z));
    ga.ddt[t * H + h] = gdt;
    pA = vdl[tid] * vdcs[tid];
    pb = gdt;
  }
  const float sA = block_sum(pA, red);
  const float sb = block_sum(pb, red);
  const float sD = block_sum(dDp, red);
  if (tid == 0) {
    atomicAdd(ga.dA + h, sA);
    if (ga.ddt_bias) atomicAdd(ga.ddt_bias + h, sb);
    if (ga.dD) atomicAdd(ga.dD + h, sD);
  }
}

size_t kb_chunk_smem() { return sizeof(float) * (6 * (size_t)kTileF + 6 * 64 + 8); }

}  // namespace

size_t bwd_workspace_bytes(const Geom& g) {
  const size_t NP = (size_t)g.N * g.P;
  return align256(simt_workspace_bytes(g)) + align256(sizeof(float) * (size_t)g.nchunks_max * g.H * NP) +
         align256(sizeof(float) * (size_t)g.ndocs * g.H * NP);
}

cudaError_t bwd_run(const Geom& g, const Args& a_in, const GradArgs& ga, void* base, int* status,
                    cudaStream_t stream) {
  const bool tc = bwd_tc_eligible(g, a_in, ga);
  if (g.Q != (tc ? kBwdTcQ : kBwdQ)) return cudaErrorInvalidValue;
  const size_t NP = (size_t)g.N * g.P;
  SimtWorkspace ws;
  simt_carve_workspace(g, base, &ws);
  char* p = static_cast<char*>(base) + align256(simt_workspace_bytes(g));
  BwdWs bw;
  bw.dstates = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * (size_t)g.nchunks_max * g.H * NP);
  bw.final = reinterpret_cast<float*>(p);
  Args a = a_in;
  a.y = nullptr;
  a.final_states = bw.final;

  ZeroList zl{};
  auto zero = [&](float* q, int64_t n) {
    if (q && n > 0) {
      zl.p[zl.count] = q;
      zl.n[zl.count] = n;
      zl.first[zl.count + 1] = zl.first[zl.count] + (n + kZeroRun - 1) / kZeroRun;
      ++zl.count;
    }
  };
  zero(ga.dB, g.tokens * g.G * g.N);
  zero(ga.dC, g.tokens * g.G * g.N);
  zero(ga.dA, g.H);
  zero(ga.dD, g.H);
  zero(ga.ddt_bias, g.H);
  // the tensor-core chunk kernel adds the parts of each 64-column slice of P into ddt
  if (tc && g.P > 64) zero(ga.ddt, g.tokens * g.H);
  if (zl.count > 0) {
    const int64_t blocks = zl.first[zl.count];
    kb_zero<<<(unsigned)(blocks < 8192 ? blocks : 8192), 256, 0, stream>>>(zl);
  }
  // the chunk-state products on the tensor cores when the chunk kernel is there and N = 128
  const bool tc_states = tc && g.N == 128;
  cudaError_t e;
  if (tc_states) {
    e = simt_cumsum(g, a, ws, status, stream);
    if (e == cudaSuccess && g.nchunks_max > 0 && g.H > 0) e = bwd_states_tc(g, a, ga, ws, bw, 0, status, stream);
    if (e == cudaSuccess) e = simt_state_pass(g, a, ws, status, stream);
  } else {
    e = simt_states(g, a, ws, status, stream);
  }
  if (e != cudaSuccess) return e;
  if (g.nchunks_max > 0 && g.H > 0) {
    if (tc_states) {
      e = bwd_states_tc(g, a, ga, ws, bw, 1, status, stream);
      if (e != cudaSuccess) return e;
    } else {
      const int tiles = ((g.N + 63) / 64) * ((g.P + 63) / 64);
      kb_chunk_dstate<<<dim3((unsigned)g.nchunks_max, g.H, tiles), 256, 0, stream>>>(g, a, ga, ws, bw);
    }
  }
  if (g.ndocs > 0 && g.H > 0) {
    kb_state_pass<<<dim3(g.ndocs, g.H, (unsigned)((NP + 255) / 256)), 256, 0, stream>>>(g, a, ga, ws,
                                                                                      bw);
  }
  if (tc && g.nchunks_max > 0 && g.H > 0) return bwd_chunk_tc(g, a, ga, ws, bw, status, stream);
  if (g.nchunks_max > 0 && g.H > 0) {
    const size_t smem = kb_chunk_smem();
    e = cudaFuncSetAttribute(kb_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kb_chunk<<<dim3((unsigned)g.nchunks_max, g.H), 256, smem, stream>>>(g, a, ga, ws, bw);
  }
  return cudaGetLastError();
}

}  // namespace ssd
