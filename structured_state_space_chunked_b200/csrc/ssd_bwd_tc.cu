// ssd_bwd_tc.cu -- the per-chunk gradients of the backward pass on tcgen05.
//
// The same chunk-level derivative as ssd_bwd.cu's kb_chunk ("Transformers are SSMs",
// paperlayer.ai summary: the block decomposition of §6, differentiated), for bf16
// inputs with P a multiple of 64 and N = 64 or 128, on 128-token chunks.  One CTA of 256
// threads per (chunk, head, 64-column slice of P); threads r and r + 128 own row r of
// every 128-row accumulator, each half of its columns.  Every gradient is linear in the
// slices of the head dimension (x, dy and the state's columns enter each term once), so a
// slice's CTA computes its part of every sum over p (S1, dY Hc^T, X dE^T, <C, dC>,
// <x, gB>, <dE, S_last>) and the parts meet in the global accumulators.  Every matrix
// is staged once in shared memory as bf16 128-byte-swizzled panels and read by the
// MMAs either K-major or MN-major:
//
//   S1 = dY X^T   (t x s)   ->  W'[t][s] = exp(cs_t - cs_s) delta_s S1[t][s], s <= t
//   S2 = C B^T    (u x s)   ->  V[u][s]  = exp(cs_u - cs_s) S2[u][s],          s <= u
//   dC = W' B + diag(exp cs) dY Hc^T                         (t x n)
//   dB = W'^T C + diag(delta exp(cs_last - cs)) X dE^T       (s x n)
//   gB = V^T dY + diag(exp(cs_last - cs)) B dE               (s x p),  dx = delta gB + D dy
//
// W' carries delta_s on its columns, so W' B is the in-chunk dC and W'^T C is delta_s
// times the in-chunk sum of dB.  The two terms of each product accumulate in separate
// TMEM columns and meet in the epilogue with their row factors.  W', V and dE enter
// the MMAs as two bf16 operands each, hi = bf16(v) and lo = bf16(v - hi): dA sums
// differences of large terms over a chunk, and a single bf16 rounding of those three
// matrices moves it by tens of per cent, while the split keeps about 16 bits.  Hc, a
// single rounding, moves dA by under 1 %.  Products run one phase at a time (S1 and S2;
// dC; dB; gB), each followed by its epilogue; every wait is bounded and reports
// SSD_ERR_TIMEOUT through the status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_bwd.h"
#include "ssd_chunks.cuh"
#include "tc_common.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kQ = kBwdTcQ;  // 128 tokens per chunk
constexpr uint32_t kTmemCols = 512;

struct TcParams {
  Geom g;
  Args a;
  GradArgs ga;
  SimtWorkspace ws;
  BwdWs bw;
  int* status;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int* status) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > 2000000000ull) {
      set_status(status, SSD_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// four fp32 additions into 16-byte-aligned global memory, one reduction instruction
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// v ~ hi + lo in bf16: two packed pairs
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  lo = pack_bf16(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

// 8 bf16 values (columns c8*8 .. c8*8+7) of row r
__device__ __forceinline__ void ld_bf16x8(uint32_t base, uint32_t panel_bytes, int r, int c8, float* out) {
  const uint4 q = ld_shared_v4(base + (uint32_t)(c8 >> 3) * panel_bytes + swz((uint32_t)r, (uint32_t)(c8 & 7)));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    out[2 * k] = __uint_as_float(w[k] << 16);
    out[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

__global__ void __launch_bounds__(256, 1) kb_chunk_tc(const __grid_constant__ CUtensorMap tm_x,
                                                   const __grid_constant__ CUtensorMap tm_dy,
                                                   const __grid_constant__ CUtensorMap tm_b,
                                                   const __grid_constant__ CUtensorMap tm_c,
                                                   const __grid_constant__ TcParams kp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tslot;
  __shared__ float vcs2[kQ], vdl[kQ], vecs[kQ], veq[kQ], vdcs[kQ], vxg[kQ];
  __shared__ float red[8];
  __shared__ float vpart[2][kQ];
  const Geom& g = kp.g;
  // 256 threads: thread (r, half) owns row r of the accumulators and half of the columns
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = tid & (kQ - 1), half = tid >> 7;
  const int64_t k = blockIdx.x;
  // blockIdx.y: (head, 64-column slice of its head dimension)
  const int nps = g.P / 64, h = (int)blockIdx.y / nps, pofs = ((int)blockIdx.y % nps) * 64;
  ChunkInfo ci;
  if (!chunk_info(g, kp.a.cu, kp.ws, k, &ci)) return;
  const int N = g.N, P = g.P, H = g.H, G = g.G, grp = h / (H / G), len = ci.len;
  const int np = N / 64;  // 64-column panels of B, C
  const int64_t NP = (int64_t)N * P, t0 = ci.start;

  // shared memory: X, dY (128 x 64), B, C (128 x N), W' then V as hi and lo (128 x 128
  // each), Hc, dE hi and lo (N x 64)
  const uint32_t sbase = (su32(smem_raw) + 1023u) & ~1023u;
  const uint32_t s_x = sbase, s_dy = s_x + kPanel, s_b = s_dy + kPanel;
  const uint32_t s_c = s_b + np * kPanel, s_w = s_c + np * kPanel, s_wl = s_w + 2 * kPanel;
  const uint32_t s_hc = s_wl + 2 * kPanel, s_de = s_hc + (uint32_t)N * 128u;
  const uint32_t s_del = s_de + (uint32_t)N * 128u;
  const uint32_t bar_load = su32(&bars[0]), bar_mma = su32(&bars[1]);

  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
    // X, dY, B and C load while the threads convert the states below
    mbar_expect_tx(bar_load, (uint32_t)(2 + 2 * np) * kPanel);
    tma_2d(s_x, &tm_x, bar_load, h * P + pofs, (int)t0);
    tma_2d(s_dy, &tm_dy, bar_load, h * P + pofs, (int)t0);
    for (int q = 0; q < np; ++q) {
      tma_3d(s_b + q * kPanel, &tm_b, bar_load, 64 * q, grp, (int)t0);
      tma_3d(s_c + q * kPanel, &tm_c, bar_load, 64 * q, grp, (int)t0);
    }
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tslot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  const int64_t cso = ((int64_t)h * g.nchunks_max + k) * g.Q;
  const float cs_last = kp.ws.cs[cso + g.Q - 1];
  if (tid < kQ) {
    const float c = kp.ws.cs[cso + tid];
    vcs2[tid] = c * 1.4426950408889634f;  // log2 units for the in-chunk decay factors
    vdl[tid] = kp.ws.delta[cso + tid];
    vecs[tid] = expf(c);
    veq[tid] = expf(cs_last - c);
    vdcs[tid] = 0.f;
    vxg[tid] = 0.f;
  }
  // the entering state and the end-of-chunk cotangent as bf16 operands (rows n)
  const float* Hc = kp.ws.states + (k * H + h) * NP;
  const float* dE = kp.bw.dstates + (k * H + h) * NP;
  // the state after the chunk (the next chunk's entering state, or the final state),
  // for <dE, S_last>, summed here over this thread's elements while dE is in registers
  int64_t first;
  const int64_t cnt = doc_chunks(g, kp.ws, ci.doc, &first);
  const float* Hend = (k == first + cnt - 1) ? kp.bw.final + ((int64_t)ci.doc * H + h) * NP
                                             : kp.ws.states + ((k + 1) * H + h) * NP;
  float sp = 0.f;
  // every (row, 8 columns) piece of this thread (N * 8 / 256 of them: 4 for N = 128, 2 for
  // N = 64) in one round, all loads issued before the stores
  {
    constexpr int kU = 4;
    float4 hv[kU][2], ev[kU][2], sv[kU][2];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = u * 256 + tid, n = i >> 3, c = i & 7;
      if (i < N * 8) {
        const int64_t off = (int64_t)n * P + pofs + 8 * c;
        const float4* ph = reinterpret_cast<const float4*>(Hc + off);
        const float4* pe = reinterpret_cast<const float4*>(dE + off);
        const float4* ps = reinterpret_cast<const float4*>(Hend + off);
        hv[u][0] = __ldg(ph);
        hv[u][1] = __ldg(ph + 1);
        ev[u][0] = __ldg(pe);
        ev[u][1] = __ldg(pe + 1);
        sv[u][0] = __ldg(ps);
        sv[u][1] = __ldg(ps + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = u * 256 + tid, n = i >> 3, c = i & 7;
      if (i >= N * 8) continue;
      const float4 h0 = hv[u][0], h1 = hv[u][1], e0 = ev[u][0], e1 = ev[u][1];
      const float4 s0 = sv[u][0], s1 = sv[u][1];
      sp += e0.x * s0.x + e0.y * s0.y + e0.z * s0.z + e0.w * s0.w + e1.x * s1.x + e1.y * s1.y +
            e1.z * s1.z + e1.w * s1.w;
      st_shared_v4(s_hc + swz((uint32_t)n, (uint32_t)c), pack_bf16(h0.x, h0.y), pack_bf16(h0.z, h0.w),
                   pack_bf16(h1.x, h1.y), pack_bf16(h1.z, h1.w));
      uint32_t eh[4], el[4];
      split2(e0.x, e0.y, eh[0], el[0]);
      split2(e0.z, e0.w, eh[1], el[1]);
      split2(e1.x, e1.y, eh[2], el[2]);
      split2(e1.z, e1.w, eh[3], el[3]);
      st_shared_v4(s_de + swz((uint32_t)n, (uint32_t)c), eh[0], eh[1], eh[2], eh[3]);
      st_shared_v4(s_del + swz((uint32_t)n, (uint32_t)c), el[0], el[1], el[2], el[3]);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  bool ok = true;
  uint32_t mma_phase = 0;

  // phase A: once the loads landed, S1 = dY X^T (cols 0..127) and S2 = C B^T (cols 256..383, kept
  // until phase D)
  if (tid == 0) {
    if (wait_bar(bar_load, 0, kp.status)) {
      tc_fence_after();
      const uint32_t id = idesc(128, 128, 0, 0);
      for (int kk = 0; kk < 4; ++kk)
        tc_mma(tmem, sdesc(s_dy + kk * 32, 16, 1024), sdesc(s_x + kk * 32, 16, 1024), id, kk > 0);
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
        tc_mma(tmem + 256, sdesc(s_c + off, 16, 1024), sdesc(s_b + off, 16, 1024), id, kk > 0);
      }
    } else {
      ok = false;
    }
    tc_commit(bar_mma);
  }
  ok = wait_bar(bar_load, 0, kp.status) && ok;
  ok = wait_bar(bar_mma, mma_phase, kp.status) && ok;
  mma_phase ^= 1u;
  tc_fence_after();

  // E1: W' rows (hi and lo), the dD diagonal
  float dDp = 0.f;
  {
    const bool row = r < len;
    const float csr2 = vcs2[r];
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
      float s1[32];
      tc_ld32(trow + c0, s1);
      tc_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float a2[2];
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const int j = 8 * q + 2 * m + z, s = c0 + j;
            const bool in = row && s <= r;
            a2[z] = in ? ex2(csr2 - vcs2[s]) * vdl[s] * s1[j] : 0.f;
            if (s == r && row) dDp = s1[j];
          }
          split2(a2[0], a2[1], wh[m], wl[m]);
        }
        const int c8 = (c0 >> 3) + q;  // 8-column group 0..15
        const uint32_t off = (uint32_t)(c8 >> 3) * kPanel + swz((uint32_t)r, (uint32_t)(c8 & 7));
        st_shared_v4(s_w + off, wh[0], wh[1], wh[2], wh[3]);
        st_shared_v4(s_wl + off, wl[0], wl[1], wl[2], wl[3]);
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();

  // phase B: dC = W' B (cols 0..N-1) and dY Hc^T (cols N..2N-1)
  if (ok && tid == 0) {
    const uint32_t idB = idesc(128, N, 0, 1), idI = idesc(128, N, 0, 0);
    for (int kk = 0; kk < 16; ++kk) {
      const uint32_t wa = ((kk & 8) ? s_wl : s_w) + ((kk >> 2) & 1) * kPanel + (kk & 3) * 32;
      tc_mma(tmem, sdesc(wa, 16, 1024), sdesc(s_b + (kk & 7) * 2048, kPanel, 1024), idB, kk > 0);
    }
    for (int kk = 0; kk < 4; ++kk)
      tc_mma(tmem + N, sdesc(s_dy + kk * 32, 16, 1024), sdesc(s_hc + kk * 32, 16, 1024), idI, kk > 0);
    tc_commit(bar_mma);
  }
  if (ok) {
    ok = wait_bar(bar_mma, mma_phase, kp.status);
    mma_phase ^= 1u;
  }
  tc_fence_after();
  // E2: dC (atomics over the group's heads) and <C_t, dC_t>
  if (ok) {
    float part = 0.f;
    for (int c0 = half * (N / 2); c0 < (half + 1) * (N / 2); c0 += 32) {
      float a[32], b[32];
      tc_ld32(trow + c0, a);
      tc_ld32(trow + N + c0, b);
      tc_wait_ld();
      if (r < len) {
        float* dst = kp.ga.dC + ((t0 + r) * G + grp) * (int64_t)N + c0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float cv[8], dc[8];
          ld_bf16x8(s_c, kPanel, r, (c0 >> 3) + q, cv);
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            const int j = 8 * q + z;
            dc[z] = fmaf(vecs[r], b[j], a[j]);
            part = fmaf(cv[z], dc[z], part);
          }
          red_add4(dst + 8 * q, dc[0], dc[1], dc[2], dc[3]);
          red_add4(dst + 8 * q + 4, dc[4], dc[5], dc[6], dc[7]);
        }
      }
    }
    vpart[half][r] = part;
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (tid < kQ) vdcs[tid] = vpart[0][tid] + vpart[1][tid];

  // phase C: dB = W'^T C (cols 0..N-1) and X dE^T (cols N..2N-1)
  if (ok && tid == 0) {
    const uint32_t idT = idesc(128, N, 1, 1), idI = idesc(128, N, 0, 0);
    for (int kk = 0; kk < 16; ++kk)
      tc_mma(tmem, sdesc(((kk & 8) ? s_wl : s_w) + (kk & 7) * 2048, kPanel, 1024),
             sdesc(s_c + (kk & 7) * 2048, kPanel, 1024), idT, kk > 0);
    for (int kk = 0; kk < 8; ++kk)
      tc_mma(tmem + N, sdesc(s_x + (kk & 3) * 32, 16, 1024),
             sdesc(((kk & 4) ? s_del : s_de) + (kk & 3) * 32, 16, 1024), idI, kk > 0);
    tc_commit(bar_mma);
  }
  if (ok) {
    ok = wait_bar(bar_mma, mma_phase, kp.status);
    mma_phase ^= 1u;
  }
  tc_fence_after();
  // E3: dB
  if (ok) {
    const float f2 = vdl[r] * veq[r];
    for (int c0 = half * (N / 2); c0 < (half + 1) * (N / 2); c0 += 32) {
      float a[32], b[32];
      tc_ld32(trow + c0, a);
      tc_ld32(trow + N + c0, b);
      tc_wait_ld();
      if (r < len) {
        float* dst = kp.ga.dB + ((t0 + r) * G + grp) * (int64_t)N + c0;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          red_add4(dst + j, fmaf(f2, b[j], a[j]), fmaf(f2, b[j + 1], a[j + 1]), fmaf(f2, b[j + 2], a[j + 2]),
                   fmaf(f2, b[j + 3], a[j + 3]));
      }
    }
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();

  // EV: V rows (hi and lo) from S2, into the space W' no longer needs
  if (ok) {
    const bool row = r < len;
    const float csr2 = vcs2[r];
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
      float s2[32];
      tc_ld32(trow + 256 + c0, s2);
      tc_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t vh[4], vl[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float b2[2];
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const int j = 8 * q + 2 * m + z, s = c0 + j;
            b2[z] = (row && s <= r) ? ex2(csr2 - vcs2[s]) * s2[j] : 0.f;
          }
          split2(b2[0], b2[1], vh[m], vl[m]);
        }
        const int c8 = (c0 >> 3) + q;
        const uint32_t off = (uint32_t)(c8 >> 3) * kPanel + swz((uint32_t)r, (uint32_t)(c8 & 7));
        st_shared_v4(s_w + off, vh[0], vh[1], vh[2], vh[3]);
        st_shared_v4(s_wl + off, vl[0], vl[1], vl[2], vl[3]);
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();

  // phase D: gB = V^T dY (cols 0..63) and B dE (cols 64..127)
  if (ok && tid == 0) {
    const uint32_t idT = idesc(128, 64, 1, 1), idK = idesc(128, 64, 0, 1);
    for (int kk = 0; kk < 16; ++kk)
      tc_mma(tmem, sdesc(((kk & 8) ? s_wl : s_w) + (kk & 7) * 2048, kPanel, 1024),
             sdesc(s_dy + (kk & 7) * 2048, kPanel, 1024), idT, kk > 0);
    const int nk = N / 16;
    for (int kk = 0; kk < 2 * nk; ++kk) {
      const int k2 = kk % nk;
      tc_mma(tmem + 64, sdesc(s_b + (k2 >> 2) * kPanel + (k2 & 3) * 32, 16, 1024),
             sdesc((kk < nk ? s_de : s_del) + k2 * 2048, (uint32_t)N * 128u, 1024), idK, kk > 0);
    }
    tc_commit(bar_mma);
  }
  if (ok) {
    ok = wait_bar(bar_mma, mma_phase, kp.status);
    mma_phase ^= 1u;
  }
  tc_fence_after();
  // E4: dx and <x, gB>
  if (ok) {
    const float Dh = kp.a.D ? kp.a.D[h] : 0.f;
    float part = 0.f;
    for (int c0 = half * 32; c0 < half * 32 + 32; c0 += 32) {
      float a[32], b[32];
      tc_ld32(trow + c0, a);
      tc_ld32(trow + 64 + c0, b);
      tc_wait_ld();
      if (r < len) {
        float4* dst = reinterpret_cast<float4*>(kp.ga.dx + ((t0 + r) * H + h) * (int64_t)P + pofs + c0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float xv[8], yv[8], o[8];
          ld_bf16x8(s_x, kPanel, r, (c0 >> 3) + q, xv);
          ld_bf16x8(s_dy, kPanel, r, (c0 >> 3) + q, yv);
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            const int j = 8 * q + z;
            const float gb = fmaf(veq[r], b[j], a[j]);
            o[z] = fmaf(vdl[r], gb, Dh * yv[z]);
            part = fmaf(xv[z], gb, part);
          }
          dst[2 * q] = make_float4(o[0], o[1], o[2], o[3]);
          dst[2 * q + 1] = make_float4(o[4], o[5], o[6], o[7]);
        }
      }
    }
    vpart[half][r] = part;
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (tid < kQ) vxg[tid] = vpart[0][tid] + vpart[1][tid];

  // E5: <dE, S_last>, dcs and its reverse cumsum, ddt, the per-head sums
  if (ok) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
    if (lane == 0) red[warp] = sp;
    __syncthreads();
    const float scal = red[0] + red[1] + red[2] + red[3] + red[4] + red[5] + red[6] + red[7];
    // reverse cumsum of dcs over the chunk by warp 0: four tokens per lane, then a
    // suffix scan of the lanes' totals
    if (warp == 0) {
      float d[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int l = 4 * lane + q;
        d[q] = l < len ? vdcs[l] - vdl[l] * vxg[l] + (l == len - 1 ? scal : 0.f) : 0.f;
      }
      d[2] += d[3];
      d[1] += d[2];
      d[0] += d[1];
      float tot = d[0];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_down_sync(0xffffffffu, tot, o);
        if (lane + o < 32) tot += u;
      }
      const float after = tot - d[0];  // everything in the lanes above this one
#pragma unroll
      for (int q = 0; q < 4; ++q) vdcs[4 * lane + q] = d[q] + after;
    }
    __syncthreads();
    float pA = 0.f, pb = 0.f;
    if (tid < len) {
      const int64_t t = t0 + tid;
      const float ddelta = fmaf(kp.a.A[h], vdcs[tid], vxg[tid]);
      const float z = load_f(kp.a.dt, t * H + h, g.in_bf16) + (kp.a.dt_bias ? kp.a.dt_bias[h] : 0.f);
      const float gdt = ddelta / (1.f + expf(-z));
      // every term is linear in the head-dimension slices: their parts add up
      if (nps == 1)
        kp.ga.ddt[t * H + h] = gdt;
      else
        atomicAdd(kp.ga.ddt + t * H + h, gdt);
      pA = vdl[tid] * vdcs[tid];
      pb = gdt;
    }
    float v3[3] = {pA, pb, dDp};
#pragma unroll
    for (int q = 0; q < 3; ++q) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v3[q] += __shfl_xor_sync(0xffffffffu, v3[q], o);
    }
    if (lane == 0) {
      atomicAdd(kp.ga.dA + h, v3[0]);
      if (kp.ga.ddt_bias) atomicAdd(kp.ga.ddt_bias + h, v3[1]);
      if (kp.ga.dD) atomicAdd(kp.ga.dD + h, v3[2]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// Chunk-state products on the tensor cores (N = 128, P a multiple of 64, one CTA per
// 64-column slice): D[n][p] = sum_t M[t][n] w_t V[t][p]
// with (M, V, w) = (B, x, exp(cs_last - cs_t) delta_t) for the forward's chunk states and
// (C, dy, exp(cs_t)) for the cotangent sums.  The weighted rows w_t V[t] enter as hi + lo
// bf16 pairs (about 16 bits), M as stored (bf16).  One CTA of 128 threads per (chunk,
// head); thread r scales token row r, then owns state row r of the accumulator.
__global__ void __launch_bounds__(128) kb_states_tc(const __grid_constant__ CUtensorMap tm_m,
                                                    const __grid_constant__ CUtensorMap tm_v,
                                                    const __grid_constant__ TcParams kp, int mode) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tslot;
  const Geom& g = kp.g;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t k = blockIdx.x;
  const int nps = g.P / 64, h = (int)blockIdx.y / nps, pofs = ((int)blockIdx.y % nps) * 64;
  ChunkInfo ci;
  if (!chunk_info(g, kp.a.cu, kp.ws, k, &ci)) return;
  const int P = g.P, H = g.H, G = g.G, grp = h / (H / G), len = ci.len;
  const int64_t NP = (int64_t)g.N * P, t0 = ci.start;
  const uint32_t sbase = (su32(smem_raw) + 1023u) & ~1023u;
  // the hi halves overwrite V in place (each thread reads its own row before writing it)
  const uint32_t s_m = sbase, s_v = s_m + 2 * kPanel, s_hi = s_v, s_lo = s_v + kPanel;
  const uint32_t bar_load = su32(&bars[0]), bar_mma = su32(&bars[1]);
  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tslot)),
                 "r"(64)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  if (tid == 0) {
    mbar_expect_tx(bar_load, 3 * kPanel);
    tma_3d(s_m, &tm_m, bar_load, 0, grp, (int)t0);
    tma_3d(s_m + kPanel, &tm_m, bar_load, 64, grp, (int)t0);
    tma_2d(s_v, &tm_v, bar_load, h * P + pofs, (int)t0);
  }
  const int64_t cso = ((int64_t)h * g.nchunks_max + k) * g.Q;
  float w = 0.f;
  if (tid < len) {
    const float c = kp.ws.cs[cso + tid];
    w = mode == 0 ? expf(kp.ws.cs[cso + g.Q - 1] - c) * kp.ws.delta[cso + tid] : expf(c);
  }
  bool ok = wait_bar(bar_load, 0, kp.status);
  // the weighted row of token tid, split into hi and lo
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float v[8];
    ld_bf16x8(s_v, kPanel, tid, c, v);
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) split2(w * v[2 * m], w * v[2 * m + 1], hi[m], lo[m]);
    const uint32_t off = swz((uint32_t)tid, (uint32_t)c);
    st_shared_v4(s_hi + off, hi[0], hi[1], hi[2], hi[3]);
    st_shared_v4(s_lo + off, lo[0], lo[1], lo[2], lo[3]);
  }
  fence_async_smem();
  tc_fence_before();
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (ok && tid == 0) {
    const uint32_t id = idesc(128, 64, 1, 1);
    for (int kk = 0; kk < 16; ++kk)
      tc_mma(tmem, sdesc(s_m + (kk & 7) * 2048, kPanel, 1024),
             sdesc(((kk & 8) ? s_lo : s_hi) + (kk & 7) * 2048, kPanel, 1024), id, kk > 0);
    tc_commit(bar_mma);
  }
  if (ok) ok = wait_bar(bar_mma, 0, kp.status);
  tc_fence_after();
  if (ok) {
    float* out = (mode == 0 ? kp.ws.states : kp.bw.dstates) + (k * H + h) * NP + (int64_t)tid * P + pofs;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < 64; c0 += 32) {
      float a[32];
      tc_ld32(trow + c0, a);
      tc_wait_ld();
      float4* o4 = reinterpret_cast<float4*>(out + c0);
#pragma unroll
      for (int q = 0; q < 8; ++q) o4[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(64) : "memory");
  }
}

size_t kb_chunk_tc_smem(int N) {
  return 1024 + (size_t)kPanel * (2 + 2 * (N / 64) + 4) + (size_t)3 * N * 128;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

bool bwd_tc_eligible(const Geom& g, const Args& a, const GradArgs& ga) {
  return g.in_bf16 && g.out_bf16 && g.P % 64 == 0 && g.P <= 256 && (g.N == 64 || g.N == 128) && aligned16(a.x) &&
         aligned16(a.B) && aligned16(a.C) && aligned16(ga.dy) && aligned16(ga.dx) &&
         aligned16(ga.dB) && aligned16(ga.dC) && g.tokens <= 0x7fffffffLL;
}

cudaError_t bwd_chunk_tc(const Geom& g, const Args& a, const GradArgs& ga, const SimtWorkspace& ws,
                         const BwdWs& bw, int* status, cudaStream_t stream) {
  if (g.Q != kQ) return cudaErrorInvalidValue;
  CUtensorMap tm_x, tm_dy, tm_b, tm_c;
  const cuuint64_t T = (cuuint64_t)g.tokens;
  {
    const cuuint64_t row = (cuuint64_t)g.H * g.P;
    const cuuint64_t dims[2] = {row, T};
    const cuuint64_t str[1] = {row * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kQ};
    if (!tc::encode_bf16_sw128(&tm_x, a.x, 2, dims, str, box)) return cudaErrorInvalidValue;
    if (!tc::encode_bf16_sw128(&tm_dy, ga.dy, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)g.N, (cuuint64_t)g.G, T};
    const cuuint64_t str[2] = {(cuuint64_t)g.N * 2, (cuuint64_t)g.G * g.N * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kQ};
    if (!tc::encode_bf16_sw128(&tm_b, a.B, 3, dims, str, box)) return cudaErrorInvalidValue;
    if (!tc::encode_bf16_sw128(&tm_c, a.C, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  TcParams kp{g, a, ga, ws, bw, status};
  const size_t smem = kb_chunk_tc_smem(g.N);
  cudaError_t e = cudaFuncSetAttribute(kb_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kb_chunk_tc<<<dim3((unsigned)g.nchunks_max, g.H * (g.P / 64)), 256, smem, stream>>>(tm_x, tm_dy, tm_b, tm_c,
                                                                                     kp);
  return cudaGetLastError();
}

}  // namespace ssd

namespace ssd {

cudaError_t bwd_states_tc(const Geom& g, const Args& a, const GradArgs& ga, const SimtWorkspace& ws,
                          const BwdWs& bw, int mode, int* status, cudaStream_t stream) {
  if (g.Q != kQ || g.N != 128 || g.P % 64 != 0) return cudaErrorInvalidValue;
  CUtensorMap tm_m, tm_v;
  const cuuint64_t T = (cuuint64_t)g.tokens;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)g.N, (cuuint64_t)g.G, T};
    const cuuint64_t str[2] = {(cuuint64_t)g.N * 2, (cuuint64_t)g.G * g.N * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kQ};
    if (!tc::encode_bf16_sw128(&tm_m, mode == 0 ? a.B : a.C, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t row = (cuuint64_t)g.H * g.P;
    const cuuint64_t dims[2] = {row, T};
    const cuuint64_t str[1] = {row * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kQ};
    if (!tc::encode_bf16_sw128(&tm_v, mode == 0 ? a.x : ga.dy, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  TcParams kp{g, a, ga, ws, bw, status};
  const size_t smem = 1024 + 4 * (size_t)kPanel;  // three CTAs per SM
  cudaError_t e = cudaFuncSetAttribute(kb_states_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kb_states_tc<<<dim3((unsigned)g.nchunks_max, g.H * (g.P / 64)), 128, smem, stream>>>(tm_m, tm_v, kp, mode);
  return cudaGetLastError();
}

}  // namespace ssd
