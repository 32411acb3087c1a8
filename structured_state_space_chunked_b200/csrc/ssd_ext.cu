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
// denominator, a scan with a single column, has chunk kernels of its own.
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

// The elementwise maps (SiLU, ReLU, identity) on B and C in one launch (blockIdx.y picks
// the array), 16 bytes per thread and step; same arithmetic and rounding as fmap_kernel.
__device__ __forceinline__ float fmap_ew(int kind, float u) {
  if (kind == SSD_FMAP_SILU) return u / (1.f + expf(-u));
  if (kind == SSD_FMAP_RELU) return fmaxf(u, 0.f);
  return u;
}

template <typename T>
__global__ void fmap_ew_kernel(int kind, int64_t nvec, const void* s0, void* d0, const void* s1, void* d1) {
  const uint4* src = reinterpret_cast<const uint4*>(blockIdx.y ? s1 : s0);
  uint4* dst = reinterpret_cast<uint4*>(blockIdx.y ? d1 : d0);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint4 q = src[i];
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h[k]);
        h[k] = __floats2bfloat162_rn(fmap_ew(kind, f.x), fmap_ew(kind, f.y));
      }
    } else {
      q.x = __float_as_uint(fmap_ew(kind, __uint_as_float(q.x)));
      q.y = __float_as_uint(fmap_ew(kind, __uint_as_float(q.y)));
      q.z = __float_as_uint(fmap_ew(kind, __uint_as_float(q.z)));
      q.w = __float_as_uint(fmap_ew(kind, __uint_as_float(q.w)));
    }
    dst[i] = q;
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
    if (D && in_bf16) {
      const uint4 q = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(x) + e0);
      const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(q2[k]);
        xv[2 * k] = f.x;
        xv[2 * k + 1] = f.y;
      }
    } else if (D) {
      const float4* q = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + e0);
      const float4 a = q[0], b = q[1];
      xv[0] = a.x, xv[1] = a.y, xv[2] = a.z, xv[3] = a.w, xv[4] = b.x, xv[5] = b.y, xv[6] = b.z, xv[7] = b.w;
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
// entering state and writes den.  For N <= 256 steps 1 and 3 take the block form
// (den_chunk_gram_kernel below); past that, this kernel runs the recurrence itself with
// one warp per (chunk, head): lane l holds state elements l, l + 32, ..., and the
// per-token dot products of step 3 are summed 32 tokens at a time through shared memory.
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

// Steps (1) and (3) in the block form of §6, for N <= 256.  One CTA of 256 threads
// per (chunk, block of up to 8 heads of one B/C group); warp w owns head w of the block
// for the per-head scans.  With cs the in-chunk cumsum of delta A (inclusive):
//   (1) z_end = sum_s exp(cs_last - cs_s) delta_s B_s, a weighted column sum of B;
//   (3) den_t = exp(cs_t) <C_t, z_in> + sum_{s<=t} exp(cs_t - cs_s) delta_s G[t][s],
//       with the chunk's Gram matrix G[t][s] = <C_t, B_s> formed once for all its heads.
// Both are the recurrence z_t = exp(delta_t A) z_{t-1} + delta_t B_t summed in another
// order.
constexpr int kGramMaxN = 256;
constexpr int kDenHeads = 8;
constexpr int kGramThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int gram_stride(int N) { return ((N + 31) & ~31) + 4; }

__device__ __forceinline__ void store_f4(float* d, uint4 q, float) {
  *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(q.x), __uint_as_float(q.y),
                                              __uint_as_float(q.z), __uint_as_float(q.w));
}
// Rows t < len (columns n < N) of a chunk's B (and C when TWO) into dst[t][n] as fp32,
// zeros elsewhere in [64][NR].  Loads are issued in batches before any of them is
// stored; 16-byte loads when vec (N a whole number of them and 16-byte-aligned bases).
template <bool TWO, typename TIn>
__device__ __forceinline__ void stage_chunk_rows(float* dB, float* dC, int NS, const TIn* B, const TIn* C,
                                                 int64_t row0, int64_t rstride, int len, int N, int NR,
                                                 int vec, int tid) {
  if (vec) {
    constexpr int V = 16 / sizeof(TIn), R = 4;
    const int vpr = NR / V, total = kDenQ * vpr;
    for (int base = tid; base < total; base += kGramThreads * R) {
      uint4 qb[R], qc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int i = base + r * kGramThreads, t = i / vpr, c = (i % vpr) * V;
        qb[r] = make_uint4(0u, 0u, 0u, 0u);
        qc[r] = qb[r];
        if (i < total && t < len && c < N) {
          const int64_t off = row0 + t * rstride + c;
          qb[r] = *reinterpret_cast<const uint4*>(B + off);
          if (TWO) qc[r] = *reinterpret_cast<const uint4*>(C + off);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int i = base + r * kGramThreads, t = i / vpr, c = (i % vpr) * V;
        if (i < total) {
          store_f4(dB + t * NS + c, qb[r], TIn());
          if (TWO) store_f4(dC + t * NS + c, qc[r], TIn());
        }
      }
    }
  } else {
    constexpr int R = 8;
    const int total = kDenQ * NR;
    for (int base = tid; base < total; base += kGramThreads * R) {
      float vb[R], vc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int i = base + r * kGramThreads, t = i / NR, n = i % NR;
        vb[r] = 0.f;
        vc[r] = 0.f;
        if (i < total && t < len && n < N) {
          vb[r] = (float)B[row0 + t * rstride + n];
          if (TWO) vc[r] = (float)C[row0 + t * rstride + n];
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int i = base + r * kGramThreads, t = i / NR, n = i % NR;
        if (i < total) {
          dB[t * NS + n] = vb[r];
          if (TWO) dC[t * NS + n] = vc[r];
        }
      }
    }
  }
}

// bf16 staging stride (elements): 16-byte rows offset by one bank quad, so the eight row
// addresses of an ldmatrix fall in distinct quads
__host__ __device__ inline int gram_stride_h(int N) { return ((N + 31) & ~31) + 8; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Rows t < len (columns n < N) of a chunk's matrix into d[t][n] as bf16, zeros elsewhere in
// [64][NR].  vec: asynchronous 16-byte copies (zero-filled past the rows and columns), all
// in flight at once, completed by the caller's cp_async_wait_all; else element copies.
__device__ __forceinline__ void stage_rows_h(__nv_bfloat16* d, int NSh, const __nv_bfloat16* src, int64_t row0,
                                             int64_t rstride, int len, int N, int NR, int vec, int tid) {
  if (vec) {
    const int vpr = NR / 8, total = kDenQ * vpr;
    const uint32_t d0 = static_cast<uint32_t>(__cvta_generic_to_shared(d));
    for (int i = tid; i < total; i += kGramThreads) {
      const int t = i / vpr, c = (i % vpr) * 8;
      const bool ok = t < len && c < N;
      cp_async16(d0 + (uint32_t)((t * NSh + c) * 2), ok ? src + row0 + t * rstride + c : src, ok ? 16 : 0);
    }
  } else {
    const __nv_bfloat16 zero = __float2bfloat16(0.f);
    for (int i = tid; i < kDenQ * NR; i += kGramThreads) {
      const int t = i / NR, n = i % NR;
      d[t * NSh + n] = (t < len && n < N) ? src[row0 + t * rstride + n] : zero;
    }
  }
}

__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// a pair of fp32 values as bf16 hi and lo halves (about 16 significant bits together)
__device__ __forceinline__ void split_pair(float2 v, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  const float2 r = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(v.x - r.x, v.y - r.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bytes of the staged B rows (bf16 pass 3): G is written over them once they are read
__host__ __device__ inline size_t den_gram_rows_h(int N) {
  const size_t rows = (size_t)kDenQ * gram_stride_h(N) * 2, g = (size_t)kDenQ * (kDenQ + 1) * 4;
  return rows > g ? rows : g;
}

size_t den_gram_smem(int N, bool out, bool bf16) {
  const size_t NS = (size_t)gram_stride(N);
  size_t f = 2 * (size_t)kDenHeads * kDenQ;  // delta, cs
  if (!out) {
    const size_t rows = bf16 ? (size_t)kDenQ * gram_stride_h(N) * 2 : (size_t)kDenQ * NS * 4;
    return rows + (f + (size_t)kDenHeads * kDenQ + (size_t)kDenHeads * kGramThreads) * 4;
  }
  f += (size_t)kDenQ * (kDenQ + 1) + (size_t)kDenQ * kDenHeads;  // G, <C, z_in>
  if (bf16) return (2 * (size_t)kDenHeads * kDenQ + (size_t)kDenHeads * NS) * 4 + den_gram_rows_h(N) +
                   (size_t)kDenQ * gram_stride_h(N) * 2;
  return (f + (size_t)(2 * kDenQ + kDenHeads) * NS) * 4;
}

template <bool OUT, typename TIn>
__global__ void __launch_bounds__(kGramThreads)
    den_chunk_gram_kernel(Geom g, const int32_t* cu, SimtWorkspace ws, const void* dt,
                          const float* A, const float* dt_bias, const void* B, const void* C,
                          float* den, int vec) {
  extern __shared__ __align__(16) unsigned char den_smem[];
  constexpr bool kH = sizeof(TIn) == 2;
  const int N = g.N, NR = (N + 31) & ~31, NS = gram_stride(N), tid = threadIdx.x, w = tid >> 5,
            lane = tid & 31;
  // the head blocks of one chunk are consecutive blocks, so they run together and share
  // the chunk's B and C rows in L2
  const int hpg = g.H / g.G, hblocks = (hpg + kDenHeads - 1) / kDenHeads, nhb = g.G * hblocks;
  const int64_t lin = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
  const int64_t k = lin / nhb;
  const int hb = (int)(lin % nhb), grp = hb / hblocks, hb0 = (hb % hblocks) * kDenHeads;
  const int nh = min(kDenHeads, hpg - hb0), h0 = grp * hpg + hb0;
  ChunkInfo ci;
  if (!chunk_info(g, cu, ws, k, &ci)) return;
  const int len = ci.len;
  float* sdl = reinterpret_cast<float*>(den_smem);  // [8][64] delta
  float* scs = sdl + kDenHeads * kDenQ;             // [8][64] cs
  float* rest = scs + kDenHeads * kDenQ;
  const int64_t row0 = (ci.start * g.G + grp) * (int64_t)N, rstride = (int64_t)g.G * N;
  const TIn* Bp = reinterpret_cast<const TIn*>(B);
  const TIn* Cp = reinterpret_cast<const TIn*>(C);

  // dt of this warp's head, loaded before the chunk rows so that both are in flight
  const int h = h0 + w;
  float r0 = 0.f, r1 = 0.f, a_h = 0.f, bias = 0.f;
  if (w < nh) {
    a_h = A[h];
    bias = dt_bias ? dt_bias[h] : 0.f;
    if (lane < len) r0 = load_f(dt, (ci.start + lane) * g.H + h, g.in_bf16);
    if (lane + 32 < len) r1 = load_f(dt, (ci.start + lane + 32) * g.H + h, g.in_bf16);
  }

  // pointers of the (OUT) products
  float* sG = nullptr;   // [64 (s)][65]: G transposed
  float* sCz = nullptr;  // [64][8]: <C_t, z_in>
  float* sZ = nullptr;   // the heads' entering states, [8][NR] (bf16) or rows 64..71 of sB (fp32)
  float* sB = nullptr;
  float* sC = nullptr;
  float* sW = nullptr;  // (pass 1) after the staged rows
  __nv_bfloat16* sBh = nullptr;
  __nv_bfloat16* sCh = nullptr;
  const int NSh = gram_stride_h(N);
  if constexpr (!OUT) {
    if constexpr (kH) {
      sBh = reinterpret_cast<__nv_bfloat16*>(rest);
      sW = reinterpret_cast<float*>(sBh + kDenQ * NSh);
      stage_rows_h(sBh, NSh, reinterpret_cast<const __nv_bfloat16*>(B), row0, rstride, len, N, NR, vec, tid);
      cp_async_wait_all();
    } else {
      sB = rest;
      sW = sB + kDenQ * NS;
      stage_chunk_rows<false>(sB, nullptr, NS, Bp, Bp, row0, rstride, len, N, NR, vec, tid);
    }
  } else {
    if constexpr (kH) {
      // sZ [8][NS], then the B rows (G over them once read), then the C rows (<C, z_in> over them)
      sZ = rest;
      sBh = reinterpret_cast<__nv_bfloat16*>(sZ + kDenHeads * NS);
      sCh = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<unsigned char*>(sBh) + den_gram_rows_h(N));
      sG = reinterpret_cast<float*>(sBh);
      sCz = reinterpret_cast<float*>(sCh);
      stage_rows_h(sBh, NSh, reinterpret_cast<const __nv_bfloat16*>(B), row0, rstride, len, N, NR, vec, tid);
      stage_rows_h(sCh, NSh, reinterpret_cast<const __nv_bfloat16*>(C), row0, rstride, len, N, NR, vec, tid);
      if (vec) {
        // the entering states, 4 floats per copy (N is a multiple of 8 here)
        const int zpr = NR / 4;
        const uint32_t z0 = static_cast<uint32_t>(__cvta_generic_to_shared(sZ));
        for (int i = tid; i < kDenHeads * zpr; i += kGramThreads) {
          const int hh = i / zpr, c = (i % zpr) * 4;
          const bool ok = hh < nh && c < N;
          cp_async16(z0 + (uint32_t)((hh * NS + c) * 4),
                     ok ? ws.states + (k * g.H + h0 + hh) * (int64_t)N + c : ws.states, ok ? 16 : 0);
        }
      } else {
        for (int i = tid; i < kDenHeads * NR; i += kGramThreads) {
          const int hh = i / NR, n = i % NR;
          sZ[hh * NS + n] = (hh < nh && n < N) ? ws.states[(k * g.H + h0 + hh) * (int64_t)N + n] : 0.f;
        }
      }
      cp_async_wait_all();
    } else {
      sG = rest;
      sCz = sG + kDenQ * (kDenQ + 1);
      float* after = sCz + kDenQ * kDenHeads;
      sB = after;                          // [64 + 8][NS]: B rows, then the entering states
      sC = sB + (kDenQ + kDenHeads) * NS;  // [64][NS]
      sZ = sB + kDenQ * NS;
      stage_chunk_rows<true>(sB, sC, NS, Bp, Cp, row0, rstride, len, N, NR, vec, tid);
      for (int i = tid; i < kDenHeads * NR; i += kGramThreads) {
        const int hh = i / NR, n = i % NR;
        sZ[hh * NS + n] = (hh < nh && n < N) ? ws.states[(k * g.H + h0 + hh) * (int64_t)N + n] : 0.f;
      }
    }
  }

  // per-head delta and inclusive cumsum (zero past the chunk's tokens)
  if (w < nh) {
    const float d0 = lane < len ? softplus_f(r0 + bias) : 0.f;
    const float d1 = lane + 32 < len ? softplus_f(r1 + bias) : 0.f;
    float c0 = d0 * a_h, c1 = d1 * a_h;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u0 = __shfl_up_sync(0xffffffffu, c0, o), u1 = __shfl_up_sync(0xffffffffu, c1, o);
      if (lane >= o) c0 += u0, c1 += u1;
    }
    c1 += __shfl_sync(0xffffffffu, c0, 31);
    if constexpr (OUT) {
      // log2 units: scs = cs log2 e for the token side, sdl = cs log2 e - log2 delta for the
      // source side (+inf past the chunk's tokens), so a decay weight is ex2(scs_t - sdl_s)
      c0 *= kLog2e;
      c1 *= kLog2e;
      sdl[w * kDenQ + lane] = c0 - log2f(d0);
      sdl[w * kDenQ + lane + 32] = c1 - log2f(d1);
    } else {
      sdl[w * kDenQ + lane] = d0;
      sdl[w * kDenQ + lane + 32] = d1;
    }
    scs[w * kDenQ + lane] = c0;
    scs[w * kDenQ + lane + 32] = c1;
  }
  __syncthreads();
  if constexpr (!OUT) {
    float* sw = sW;                       // [8][64] weights exp(cs_last - cs_s) delta_s
    float* red = sw + kDenHeads * kDenQ;  // [8][parts * N] partial sums
    for (int i = tid; i < kDenHeads * kDenQ; i += kGramThreads) {
      const int hh = i / kDenQ;
      sw[i] = hh < nh ? expf(scs[hh * kDenQ + kDenQ - 1] - scs[i]) * sdl[i] : 0.f;
    }
    __syncthreads();
    if constexpr (kH) {
      // z_end = B^T W on the tensor cores: warp w takes the 16-row blocks w, w + 8, ... of
      // the state dimension; A = B^T from the staged rows by transposing loads, W (tokens x
      // heads) as bf16 hi + lo
      const uint32_t aB = static_cast<uint32_t>(__cvta_generic_to_shared(sBh));
      for (int mb = w; mb < NR / 16; mb += 8) {
        float zacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < kDenQ; kk += 16) {
          uint32_t a0, a1, a2, a3, bh0, bl0, bh1, bl1;
          const int t = kk + (lane & 7) + ((lane >> 4) << 3);
          const int col = mb * 16 + (((lane >> 3) & 1) << 3);
          ldsm_x4_trans(aB + (uint32_t)((t * NSh + col) * 2), a0, a1, a2, a3);
          // B fragment of W: head lane / 4, tokens kk + 2 (lane % 4) + {0, 1} (+ 8)
          const float* wr = sw + (lane >> 2) * kDenQ + kk + 2 * (lane & 3);
          split_pair(*reinterpret_cast<const float2*>(wr), bh0, bl0);
          split_pair(*reinterpret_cast<const float2*>(wr + 8), bh1, bl1);
          mma_bf16_16816(zacc, a0, a1, a2, a3, bh0, bh1);
          mma_bf16_16816(zacc, a0, a1, a2, a3, bl0, bl1);
        }
        const int n = mb * 16 + (lane >> 2), hc = 2 * (lane & 3);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int nn = n + (q >> 1) * 8, hh = hc + (q & 1);
          if (nn < N && hh < nh) ws.states[(k * g.H + h0 + hh) * (int64_t)N + nn] = zacc[q];
        }
      }
      if (tid < nh)
        ws.cs[((int64_t)(h0 + tid) * g.nchunks_max + k) * g.Q + g.Q - 1] = scs[tid * kDenQ + kDenQ - 1];
      return;
    }
    // thread (part, n) sums tokens part, part + parts, ... of column n for every head
    const int parts = max(1, kGramThreads / N), n = tid % N, part = tid / N;
    if (part < parts) {
      float acc[kDenHeads];
#pragma unroll
      for (int hh = 0; hh < kDenHeads; ++hh) acc[hh] = 0.f;
      for (int t = part; t < len; t += parts) {
        const float bv = sB[t * NS + n];
#pragma unroll
        for (int hh = 0; hh < kDenHeads; ++hh) acc[hh] = fmaf(sw[hh * kDenQ + t], bv, acc[hh]);
      }
#pragma unroll
      for (int hh = 0; hh < kDenHeads; ++hh) red[(hh * parts + part) * N + n] = acc[hh];
    }
    __syncthreads();
    for (int i = tid; i < nh * N; i += kGramThreads) {
      const int hh = i / N, nn = i % N;
      float z = 0.f;
      for (int q = 0; q < parts; ++q) z += red[(hh * parts + q) * N + nn];
      ws.states[(k * g.H + h0 + hh) * (int64_t)N + nn] = z;
    }
    if (tid < nh) ws.cs[((int64_t)(h0 + tid) * g.nchunks_max + k) * g.Q + g.Q - 1] = scs[tid * kDenQ + kDenQ - 1];
  } else {
    if constexpr (kH) {
      // G on the tensor cores: warp w computes rows 16 (w / 2).. and columns 32 (w % 2)..
      // as four m16n8k16 tiles per 16-wide step of the state dimension.  The even warps also
      // take <C_t, z_in> of their 16 rows for the 8 heads, z split into bf16 hi + lo.
      const int t0 = (w >> 1) * 16, s0 = (w & 1) * 32;
      const bool cz = (w & 1) == 0;
      float acc[4][4], czacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
      const uint32_t aC = static_cast<uint32_t>(__cvta_generic_to_shared(sCh));
      const uint32_t aB = static_cast<uint32_t>(__cvta_generic_to_shared(sBh));
      for (int kk = 0; kk < NR; kk += 16) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(aC + (uint32_t)(((t0 + (lane & 15)) * NSh + kk + ((lane >> 4) << 3)) * 2), a0, a1, a2, a3);
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
          uint32_t b0, b1, b2, b3;
          const int srow = s0 + 16 * jp + (lane & 7) + ((lane >> 4) << 3);
          ldsm_x4(aB + (uint32_t)((srow * NSh + kk + (((lane >> 3) & 1) << 3)) * 2), b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * jp], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(acc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
        }
        if (cz) {
          // B fragment of z: head lane / 4, state elements kk + 2 (lane % 4) + {0, 1} (+ 8)
          const float* zr = sZ + (lane >> 2) * NS + kk + 2 * (lane & 3);
          uint32_t zh0, zl0, zh1, zl1;
          split_pair(*reinterpret_cast<const float2*>(zr), zh0, zl0);
          split_pair(*reinterpret_cast<const float2*>(zr + 8), zh1, zl1);
          mma_bf16_16816(czacc, a0, a1, a2, a3, zh0, zh1);
          mma_bf16_16816(czacc, a0, a1, a2, a3, zl0, zl1);
        }
      }
      __syncthreads();  // every warp has read the B and C rows that G and <C, z_in> replace
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int sc = s0 + 8 * j + 2 * (lane & 3), t = t0 + (lane >> 2);
        sG[sc * (kDenQ + 1) + t] = acc[j][0];
        sG[(sc + 1) * (kDenQ + 1) + t] = acc[j][1];
        sG[sc * (kDenQ + 1) + t + 8] = acc[j][2];
        sG[(sc + 1) * (kDenQ + 1) + t + 8] = acc[j][3];
      }
      if (cz) {
        const int t = t0 + (lane >> 2), hc = 2 * (lane & 3);
        sCz[t * kDenHeads + hc] = czacc[0];
        sCz[t * kDenHeads + hc + 1] = czacc[1];
        sCz[(t + 8) * kDenHeads + hc] = czacc[2];
        sCz[(t + 8) * kDenHeads + hc + 1] = czacc[3];
      }
    } else {
      // G[t][s] for t = ti + 16 a, s = si + 16 b: with NS = 4 (mod 32) the 16 B rows a warp
      // reads land in distinct bank quads two by two (two wavefronts per float4 read)
      const int ti = tid >> 4, si = tid & 15;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acc[a][bb] = 0.f;
      for (int n = 0; n < NR; n += 4) {
        float4 cv[4], bv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) cv[a] = *reinterpret_cast<const float4*>(sC + (ti + 16 * a) * NS + n);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) bv[bb] = *reinterpret_cast<const float4*>(sB + (si + 16 * bb) * NS + n);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) {
            float v = acc[a][bb];
            v = fmaf(cv[a].x, bv[bb].x, v);
            v = fmaf(cv[a].y, bv[bb].y, v);
            v = fmaf(cv[a].z, bv[bb].z, v);
            acc[a][bb] = fmaf(cv[a].w, bv[bb].w, v);
          }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) sG[(si + 16 * bb) * (kDenQ + 1) + ti + 16 * a] = acc[a][bb];
      const int t = tid >> 2, hp = (tid & 3) * 2;
      float c0 = 0.f, c1 = 0.f;
      for (int n = 0; n < NR; n += 4) {
        const float4 cv = *reinterpret_cast<const float4*>(sC + t * NS + n);
        const float4 z0 = *reinterpret_cast<const float4*>(sZ + hp * NS + n);
        const float4 z1 = *reinterpret_cast<const float4*>(sZ + (hp + 1) * NS + n);
        c0 = fmaf(cv.x, z0.x, fmaf(cv.y, z0.y, fmaf(cv.z, z0.z, fmaf(cv.w, z0.w, c0))));
        c1 = fmaf(cv.x, z1.x, fmaf(cv.y, z1.y, fmaf(cv.z, z1.z, fmaf(cv.w, z1.w, c1))));
      }
      sCz[t * kDenHeads + hp] = c0;
      sCz[t * kDenHeads + hp + 1] = c1;
    }
    __syncthreads();
    if (w < nh) {
      // lane l: tokens l and l + 32.  A source in the first 32-block reaches token l + 32
      // through the block boundary: exp(cs_t - cs_s) = exp(cs_t - cs_31) exp(cs_31 - cs_s),
      // both factors at most 1.  In log2 units the weight of source s at token t is
      // ex2(scs_t - sdl_s) = exp(cs_t - cs_s) delta_s.
      const float* sv = sdl + w * kDenQ;
      const float* cs = scs + w * kDenQ;
      const float c0 = cs[lane], c1 = cs[lane + 32], cm = cs[31];
      const float u = ex2a(cm - sv[lane]);
      float s0 = 0.f, s1 = 0.f;
      for (int sidx = 0; sidx < 32; ++sidx) {
        const float* gs = sG + sidx * (kDenQ + 1);
        const float us = __shfl_sync(0xffffffffu, u, sidx);
        if (sidx <= lane) s0 = fmaf(ex2a(c0 - sv[sidx]), gs[lane], s0);
        s1 = fmaf(us, gs[lane + 32], s1);
      }
      s1 *= ex2a(c1 - cm);
      for (int sidx = 32; sidx < kDenQ; ++sidx)
        if (sidx <= lane + 32) s1 = fmaf(ex2a(c1 - sv[sidx]), sG[sidx * (kDenQ + 1) + lane + 32], s1);
      s0 = fmaf(ex2a(c0), sCz[lane * kDenHeads + w], s0);
      s1 = fmaf(ex2a(c1), sCz[(lane + 32) * kDenHeads + w], s1);
      if (lane < len) den[(ci.start + lane) * g.H + h] = s0;
      if (lane + 32 < len) den[(ci.start + lane + 32) * g.H + h] = s1;
    }
  }
}

// (2): per (document, head, state element), the chunks' end states become entering
// states; sixteen chunks of loads are issued ahead of their dependent updates
__global__ void __launch_bounds__(256) den_pass_kernel(Geom g, SimtWorkspace ws) {
  const int d = blockIdx.x, h = blockIdx.y;
  const int n = blockIdx.z * 256 + threadIdx.x;
  if (n >= g.N) return;
  if (g.varlen && !ws.total_chunks[1]) return;
  int64_t first;
  const int64_t cnt = doc_chunks(g, ws, d, &first);
  float carry = 0.f;
  constexpr int kU = 16;
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

cudaError_t fmap_apply(int kind, int64_t rows, int N, int Nout, int bf16, const void* srcB, void* dstB,
                       const void* srcC, void* dstC, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int64_t total = rows * N;
  const int V = bf16 ? 8 : 4;
  const bool ew = kind == SSD_FMAP_NONE || kind == SSD_FMAP_SILU || kind == SSD_FMAP_RELU;
  const bool al = (((uintptr_t)srcB | (uintptr_t)dstB | (uintptr_t)srcC | (uintptr_t)dstC) & 15u) == 0;
  if (ew && Nout == N && al && total % V == 0) {
    const int64_t nvec = total / V;
    const dim3 grid(grid_for(nvec), 2);
    if (bf16)
      fmap_ew_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(kind, nvec, srcB, dstB, srcC, dstC);
    else
      fmap_ew_kernel<float><<<grid, 256, 0, stream>>>(kind, nvec, srcB, dstB, srcC, dstC);
    return cudaGetLastError();
  }
  fmap_kernel<<<grid_for(rows * Nout), 256, 0, stream>>>(kind, rows, N, Nout, bf16, srcB, dstB);
  fmap_kernel<<<grid_for(rows * Nout), 256, 0, stream>>>(kind, rows, N, Nout, bf16, srcC, dstC);
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
  if (g.N <= kGramMaxN) {
    // block form, one CTA per (chunk, up to 8 heads of a group)
    const int hblocks = (g.H / g.G + kDenHeads - 1) / kDenHeads;
    const dim3 grid((unsigned)g.nchunks_max, (unsigned)(g.G * hblocks));
    const int V = g.in_bf16 ? 8 : 4;
    const int vec = g.N % V == 0 && ((uintptr_t)B & 15u) == 0 && ((uintptr_t)C & 15u) == 0;
    cudaError_t e = cudaSuccess;
    auto run = [&](auto kern, bool out) {
      if (e != cudaSuccess) return;
      const size_t sm = den_gram_smem(g.N, out, g.in_bf16 != 0);
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e == cudaSuccess) {
        kern<<<grid, kGramThreads, sm, stream>>>(g, cu, ws, dt, A, dt_bias, B, C, den, vec);
        e = cudaGetLastError();
      }
    };
    if (g.in_bf16)
      run(den_chunk_gram_kernel<false, __nv_bfloat16>, false);
    else
      run(den_chunk_gram_kernel<false, float>, false);
    if (e == cudaSuccess && g.ndocs > 0) {
      den_pass_kernel<<<dim3(g.ndocs, g.H, (unsigned)((g.N + 255) / 256)), 256, 0, stream>>>(g, ws);
      e = cudaGetLastError();
    }
    if (g.in_bf16)
      run(den_chunk_gram_kernel<true, __nv_bfloat16>, true);
    else
      run(den_chunk_gram_kernel<true, float>, true);
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
