// ssd_cp.cu -- the three device steps of a context-parallel forward.
//
// A sequence is cut into consecutive slices, one per rank ("Transformers are SSMs",
// paperlayer.ai summary, §8.2: a worker passes its final state to the next; the
// state-passing scan of §6.2 across workers).  Each rank runs ssd_forward on its
// slice from a zero state, which gives its outputs and its local final state S_r
// correct except for the state that should have entered the slice.  With cs_t the
// cumulative sum of delta A over the slice up to token t and ld_r = cs_last:
//
//   H_in(0) = init;   H_in(r + 1) = exp(ld_r) H_in(r) + S_r             (scan over ranks)
//   final_r = exp(ld_r) H_in(r) + S_r
//   y_t    += exp(cs_t) C_t H_in(r)                                    (the left factors, §6.2)
//
// ssd_cp_logdecay writes cs (and ld); ssd_cp_combine runs the scan for one rank
// from every rank's (S, ld); ssd_cp_correct adds the entering state's contribution
// to y.  Batch mode only: each batch row is one sequence cut into the ranks' slices.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd_internal.h"
#include "tc_common.cuh"

namespace ssd {
namespace {

constexpr int kScanThreads = 256;

// cs[b, t, h] = sum_{k <= t} softplus(dt + dt_bias) A over the slice; ld[b, h] = cs at the
// last token.  One CTA per (b, h), the tokens in blocks of 256 with a running carry.
__global__ void __launch_bounds__(kScanThreads)
    cp_logdecay_kernel(int64_t L, int H, int in_bf16, const void* dt, const float* A,
                       const float* dt_bias, float* cs, float* ld) {
  __shared__ float warp_tot[kScanThreads / 32];
  __shared__ float carry_s;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const float a = A[h], bias = dt_bias ? dt_bias[h] : 0.f;
  if (threadIdx.x == 0) carry_s = 0.f;
  __syncthreads();
  for (int64_t t0 = 0; t0 < L; t0 += kScanThreads) {
    const int64_t t = t0 + threadIdx.x;
    float v = 0.f;
    if (t < L) v = softplus_f(load_f(dt, ((int64_t)b * L + t) * H + h, in_bf16) + bias) * a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[wid] = v;
    __syncthreads();
    float base = carry_s;
    for (int w = 0; w < wid; ++w) base += warp_tot[w];
    v += base;
    if (t < L) cs[((int64_t)b * L + t) * H + h] = v;
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry_s = v;  // inclusive sum at the block's end
    __syncthreads();
  }
  if (threadIdx.x == 0) ld[bh] = carry_s;
}

// H_in and final state of rank r from every rank's local final state and log decay.
__global__ void cp_combine_kernel(int r, int nranks, int64_t BH, int64_t NP, const float* S_all,
                                  const float* ld_all, const float* init, float* h_in,
                                  float* final_states) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BH * NP) return;
  const int64_t bh = i / NP;
  float hv = init ? init[i] : 0.f;
  for (int k = 0; k < r; ++k) hv = fmaf(expf(ld_all[k * BH + bh]), hv, S_all[k * BH * NP + i]);
  if (h_in) h_in[i] = hv;
  if (final_states) final_states[i] = fmaf(expf(ld_all[r * BH + bh]), hv, S_all[r * BH * NP + i]);
  (void)nranks;
}

// The same, four consecutive state elements per thread with 16-byte accesses (N P a
// multiple of 4 and every array 16-byte aligned); every rank's load is issued before
// the Horner updates that use it.
__device__ __forceinline__ float4 f4_fma(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__global__ void cp_combine4_kernel(int r, int64_t BH, int64_t NP, const float4* S_all, const float* ld_all,
                                   const float4* init, float4* h_in, float4* final_states) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // float4 index
  const int64_t NP4 = NP / 4;
  if (i >= BH * NP4) return;
  const int64_t bh = i / NP4;
  float4 hv = init ? __ldg(init + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  int k = 0;
  for (; k + 4 <= r; k += 4) {
    float4 s[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) s[u] = __ldg(S_all + (k + u) * BH * NP4 + i);
#pragma unroll
    for (int u = 0; u < 4; ++u) hv = f4_fma(expf(ld_all[(k + u) * BH + bh]), hv, s[u]);
  }
  for (; k < r; ++k) hv = f4_fma(expf(ld_all[k * BH + bh]), hv, __ldg(S_all + k * BH * NP4 + i));
  if (h_in) h_in[i] = hv;
  if (final_states) final_states[i] = f4_fma(expf(ld_all[r * BH + bh]), hv, __ldg(S_all + r * BH * NP4 + i));
}

// y[b, t, h, :] += exp(cs[b, t, h]) C[b, t, g, :] H_in[b, h]: one CTA per (b, h, 64 tokens);
// the state in shared memory, 4 tokens x 4 columns per thread.
constexpr int kCorrTok = 64;
__global__ void __launch_bounds__(256)
    cp_correct_kernel(int64_t L, int H, int P, int N, int G, int in_bf16, int out_bf16,
                      const void* C, const float* cs, const float* h_in, void* y) {
  extern __shared__ float sm[];  // [N][P] state, then [kCorrTok][N] C
  float* Hs = sm;
  float* Cs = sm + (size_t)N * P;
  const int64_t ntile = (L + kCorrTok - 1) / kCorrTok;
  const int64_t bh = blockIdx.x / ntile;
  const int64_t t0 = (blockIdx.x % ntile) * kCorrTok;
  const int b = (int)(bh / H), h = (int)(bh % H), g = h / (H / G);
  const int nt = (int)min((int64_t)kCorrTok, L - t0);
  for (int i = threadIdx.x; i < N * P; i += blockDim.x) Hs[i] = h_in[bh * (int64_t)N * P + i];
  for (int i = threadIdx.x; i < kCorrTok * N; i += blockDim.x) {
    const int tt = i / N, n = i % N;
    Cs[i] = tt < nt ? load_f(C, (((int64_t)b * L + t0 + tt) * G + g) * N + n, in_bf16) : 0.f;
  }
  __syncthreads();
  // thread -> 4 consecutive tokens x 4 consecutive columns
  const int pq = P / 4;
  for (int job = threadIdx.x; job < (kCorrTok / 4) * pq; job += blockDim.x) {
    const int tq = job / pq, p4 = job % pq;
    float acc[4][4] = {};
    for (int n = 0; n < N; ++n) {
      const float4 hv = *reinterpret_cast<const float4*>(Hs + (size_t)n * P + 4 * p4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float c = Cs[(4 * tq + i) * N + n];
        acc[i][0] = fmaf(c, hv.x, acc[i][0]);
        acc[i][1] = fmaf(c, hv.y, acc[i][1]);
        acc[i][2] = fmaf(c, hv.z, acc[i][2]);
        acc[i][3] = fmaf(c, hv.w, acc[i][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tt = 4 * tq + i;
      if (tt >= nt) break;
      const int64_t t = t0 + tt;
      const float e = expf(cs[((int64_t)b * L + t) * H + h]);
      const int64_t yo = (((int64_t)b * L + t) * H + h) * P + 4 * p4;
#pragma unroll
      for (int j = 0; j < 4; ++j) store_f(y, yo + j, fmaf(e, acc[i][j], load_f(y, yo + j, out_bf16)), out_bf16);
    }
  }
}

// The correction on the tensor cores (bf16 C; headdim and dstate multiples of 64 up
// to 256).  Work item = (b, h, column block of Pc <= 128 state columns, a run of
// 128-token tiles); a persistent grid strides over the items.  Per item the CTA
// writes its block of H_in once as a bf16 MN-major operand (state rows n are K).
// Per tile: TMA brings the C tile into shared memory (the next one loads while this
// tile's epilogue runs), one thread issues C H_in into TMEM (M = 128 tokens, N = Pc,
// K = dstate), two threads per token row scale their halves of its accumulator row
// by exp(cs_t) and stage them in y's type, and a TMA reduction adds the staged tile
// into y (rows past the slice are clipped).  y is never read by the CTA: the addition
// happens in L2, so no load of y sits in the tile's chain.
constexpr int kCorrTile = 128;
struct CorrParams {
  int64_t L;
  int H, P, N, G, Pc, out_bf16;
  int ntiles, chunk, items_per_unit, items;
  const float* cs;
  const float* h_in;
  int* status;
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// bounded wait on an mbarrier phase; false (and the status word set) when it ran out
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t ph, int* status) {
  const uint64_t w0 = tc::globaltimer();
  while (!tc::mbar_try(bar, ph)) {
    if (tc::globaltimer() - w0 > 2000000000ull) {
      set_status(status, SSD_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, uint32_t src, int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__global__ void __launch_bounds__(256)
    cp_correct_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                         const __grid_constant__ CorrParams p) {
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = (su32(smem_raw) + 1023u) & ~1023u;
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tslot;
  const int npanel = p.N / 64;                       // 64-wide dstate panels of a C tile
  const int es = p.out_bf16 ? 2 : 4;
  const int ycols = 128 / es;                        // y columns per 128-byte panel row
  const int ypanels = p.Pc / ycols;
  const uint32_t c_bytes = (uint32_t)npanel * kPanel, y_bytes = (uint32_t)ypanels * kPanel;
  const uint32_t off_y = c_bytes, off_hb = c_bytes + y_bytes;
  const uint32_t hb_panel = (uint32_t)p.N * 128u;    // one 64-column panel of the state block
  // 256 threads: threads r and r + 128 share token row r, each taking half the columns
  const int warp = threadIdx.x >> 5, r = threadIdx.x & 127, half = threadIdx.x >> 7;
  const int nblk = p.P / p.Pc;
  const uint32_t full = su32(&bars[0]), done = su32(&bars[1]);
  const uint32_t tcols = (uint32_t)p.Pc;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&tslot)),
                 "r"(tcols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  const uint32_t id = idesc(128, p.Pc, 0, 1);
  const uint64_t dc = sdesc(sbase, 16, 1024), dh = sdesc(sbase + off_hb, hb_panel, 1024);
  const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  // C tiles are loaded one ahead: the load of tile it (this CTA's count) completes
  // phase it of `full`; nload counts the loads issued (thread 0)
  uint32_t it = 0, nload = 0;
  bool ok = true;
  auto load_c = [&](int g, int64_t row0) {
    mbar_expect_tx(full, c_bytes);
    for (int q = 0; q < npanel; ++q) tma_3d(sbase + q * kPanel, &tm_c, full, 64 * q, g, (int)row0);
    ++nload;
  };
  for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
    const int unit = item / p.items_per_unit;        // (b, h, column block)
    const int tile0 = (item % p.items_per_unit) * p.chunk;
    const int tile1 = min(p.ntiles, tile0 + p.chunk);
    const int pb = unit % nblk, bh = unit / nblk;
    const int b = bh / p.H, h = bh % p.H, g = h / (p.H / p.G);
    // the item's first C tile loads while the state block converts (the previous
    // item's products have completed: every tile waited on `done`)
    if (threadIdx.x == 0) load_c(g, (int64_t)b * p.L + (int64_t)tile0 * kCorrTile);
    // this block of H_in as bf16: row n, 64-column panels, 128-byte swizzle
    const float* hsrc = p.h_in + (int64_t)bh * p.N * p.P + pb * p.Pc;
    for (int i = threadIdx.x; i < p.N * (p.Pc / 8); i += blockDim.x) {
      const int n = i / (p.Pc / 8), c8 = i % (p.Pc / 8);
      const float4 u = *reinterpret_cast<const float4*>(hsrc + (int64_t)n * p.P + 8 * c8);
      const float4 v = *reinterpret_cast<const float4*>(hsrc + (int64_t)n * p.P + 8 * c8 + 4);
      st_shared_v4(sbase + off_hb + (c8 >> 3) * hb_panel + swz((uint32_t)n, (uint32_t)(c8 & 7)),
                   pack_bf16(u.x, u.y), pack_bf16(u.z, u.w), pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
    }
    fence_async_smem();
    __syncthreads();
    for (int j = tile0; j < tile1 && ok; ++j, ++it) {
      const uint32_t ph = it & 1u;
      const int t0 = j * kCorrTile;
      if (threadIdx.x == 0) {
        if (wait_phase(full, ph, p.status)) {
          tc_fence_after();
          for (int kk = 0; kk < p.N / 16; ++kk)
            tc_mma(tmem, dc + (((kk >> 2) * kPanel + (kk & 3) * 32) >> 4), dh + ((kk * 2048) >> 4), id,
                   kk > 0);
        } else {
          ok = false;
        }
        tc_commit(done);  // arrives even when nothing was issued
        bulk_wait_read0();  // the previous tile's reduction has read the staging tile
      }
      ok = __syncthreads_and(ok);
      ok = wait_phase(done, ph, p.status) && ok;
      // the products have read C: the next tile's C tile loads during this epilogue
      if (threadIdx.x == 0 && ok && j + 1 < tile1) load_c(g, (int64_t)b * p.L + t0 + kCorrTile);
      tc_fence_after();
      // the correction exp(cs_t) (C_t H_in), in y's type, staged for a TMA reduction
      // (addition) into y
      const int64_t t = (int64_t)t0 + r;
      const float e = (ok && t < p.L) ? expf(p.cs[((int64_t)b * p.L + t) * p.H + h]) : 0.f;
      for (int c0 = half * (p.Pc / 2); c0 < (half + 1) * (p.Pc / 2); c0 += 32) {
        float acc[32];
        tc_ld32(ta + c0, acc);
        tc_wait_ld();
        if (p.out_bf16) {
          const uint32_t row = sbase + off_y + (c0 >> 6) * kPanel;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_shared_v4(row + swz((uint32_t)r, (uint32_t)(((c0 & 63) >> 3) + k)),
                         pack_bf16(e * acc[8 * k], e * acc[8 * k + 1]), pack_bf16(e * acc[8 * k + 2], e * acc[8 * k + 3]),
                         pack_bf16(e * acc[8 * k + 4], e * acc[8 * k + 5]),
                         pack_bf16(e * acc[8 * k + 6], e * acc[8 * k + 7]));
        } else {
          const uint32_t row = sbase + off_y + (c0 >> 5) * kPanel;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(row + swz((uint32_t)r, (uint32_t)k), __float_as_uint(e * acc[4 * k]),
                         __float_as_uint(e * acc[4 * k + 1]), __float_as_uint(e * acc[4 * k + 2]),
                         __float_as_uint(e * acc[4 * k + 3]));
        }
      }
      fence_async_smem();  // the staged tile is read by the TMA reduction
      tc_fence_before();
      ok = __syncthreads_and(ok);
      tc_fence_after();
      if (threadIdx.x == 0 && ok) {
        for (int q = 0; q < ypanels; ++q)
          tma_reduce_add_3d(&tm_y, sbase + off_y + q * kPanel, h * p.P + pb * p.Pc + q * ycols, t0, b);
        bulk_commit();
      }
    }
  }
  if (threadIdx.x == 0) {
    bulk_wait0();
    // the last C load has landed before shared memory goes (already true unless a
    // wait ran out; bounded by time only)
    if (nload > 0) wait_drain(full, (nload - 1) & 1u, 2000000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tcols) : "memory");
  }
}

// tensor map with a 128-byte swizzle for bf16 or fp32 data
bool encode_sw128(CUtensorMap* m, bool bf16, const void* base, int rank, const cuuint64_t* dims,
                  const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  static tc::EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult res;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) != cudaSuccess ||
        res != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<tc::EncodeTiledFn>(q);
  }
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank,
            const_cast<void*>(base), dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* q, size_t a) { return ((uintptr_t)q % a) == 0; }

int check_desc(const ssd_desc_t* desc) {
  if (!desc) return SSD_ERR_INVALID_ARG;
  const ssd_desc_t& d = *desc;
  if (d.batch < 0 || d.seqlen < 0 || d.max_docs != 0) return SSD_ERR_INVALID_ARG;
  if (d.nheads < 1 || d.headdim < 1 || d.dstate < 1 || d.ngroups < 1 || d.nheads % d.ngroups)
    return SSD_ERR_INVALID_ARG;
  if ((d.in_dtype != SSD_F32 && d.in_dtype != SSD_BF16) ||
      (d.out_dtype != SSD_F32 && d.out_dtype != SSD_BF16))
    return SSD_ERR_INVALID_ARG;
  if (d.batch * d.nheads > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
  return SSD_OK;
}

int launch_rc() { return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA; }

}  // namespace
}  // namespace ssd

extern "C" SSD_API int ssd_cp_logdecay(const ssd_desc_t* desc, const void* dt, const float* A,
                                       const float* dt_bias, float* cs, float* logdecay,
                                       ssd_stream_t stream) {
  ssd::NvtxRange nvtx_range("ssd_cp_logdecay");
  int rc = ssd::check_desc(desc);
  if (rc) return rc;
  const ssd_desc_t& d = *desc;
  if (d.batch == 0) return SSD_OK;
  if (!A || !cs || !logdecay || (d.seqlen > 0 && !dt)) return SSD_ERR_INVALID_ARG;
  ssd::cp_logdecay_kernel<<<(unsigned)(d.batch * d.nheads), ssd::kScanThreads, 0,
                            reinterpret_cast<cudaStream_t>(stream)>>>(
      d.seqlen, d.nheads, d.in_dtype == SSD_BF16, dt, A, dt_bias, cs, logdecay);
  return ssd::launch_rc();
}

extern "C" SSD_API int ssd_cp_combine(const ssd_desc_t* desc, int rank, int nranks,
                                      const float* local_final_all, const float* logdecay_all,
                                      const float* initial_states, float* h_in,
                                      float* final_states, ssd_stream_t stream) {
  ssd::NvtxRange nvtx_range("ssd_cp_combine");
  int rc = ssd::check_desc(desc);
  if (rc) return rc;
  const ssd_desc_t& d = *desc;
  if (nranks < 1 || rank < 0 || rank >= nranks) return SSD_ERR_INVALID_ARG;
  const int64_t BH = d.batch * d.nheads, NP = (int64_t)d.dstate * d.headdim;
  if (BH == 0) return SSD_OK;
  if (!local_final_all || !logdecay_all || (!h_in && !final_states)) return SSD_ERR_INVALID_ARG;
  const int64_t n = BH * NP;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (NP % 4 == 0 && ssd::aligned(local_final_all, 16) && ssd::aligned(initial_states, 16) &&
      ssd::aligned(h_in, 16) && ssd::aligned(final_states, 16)) {
    const int64_t n4 = n / 4;
    ssd::cp_combine4_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(
        rank, BH, NP, reinterpret_cast<const float4*>(local_final_all), logdecay_all,
        reinterpret_cast<const float4*>(initial_states), reinterpret_cast<float4*>(h_in),
        reinterpret_cast<float4*>(final_states));
    return ssd::launch_rc();
  }
  ssd::cp_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
      rank, nranks, BH, NP, local_final_all, logdecay_all, initial_states, h_in, final_states);
  return ssd::launch_rc();
}

extern "C" SSD_API int ssd_cp_correct(const ssd_desc_t* desc, const void* C, const float* cs,
                                      const float* h_in, void* y, int* status, ssd_stream_t stream) {
  ssd::NvtxRange nvtx_range("ssd_cp_correct");
  int rc = ssd::check_desc(desc);
  if (rc) return rc;
  const ssd_desc_t& d = *desc;
  if (d.batch == 0 || d.seqlen == 0) return SSD_OK;
  if (!C || !cs || !h_in || !y) return SSD_ERR_INVALID_ARG;
  if (d.headdim % 4 != 0 || !ssd::aligned(h_in, 16)) return SSD_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool tc_ok = d.in_dtype == SSD_BF16 && d.headdim % 64 == 0 && d.headdim <= 256 &&
                     d.dstate % 64 == 0 && d.dstate <= 256 && ssd::aligned(C, 16) &&
                     ssd::aligned(y, 16) && d.batch * d.seqlen <= 0x7fffffffLL &&
                     d.seqlen >= ssd::kCorrTile && d.seqlen <= 0x7fffffffLL - ssd::kCorrTile;
  if (tc_ok) {
    const bool ob = d.out_dtype == SSD_BF16;
    const int es = ob ? 2 : 4, Pc = d.headdim % 128 == 0 ? 128 : 64;  // divides headdim
    // C as [batch * L, G, N] in 64 x 1 x 128 boxes; y as [batch, L, H * P] in
    // (128 bytes) x 128 x 1 boxes; both with a 128-byte swizzle
    CUtensorMap tm_c, tm_y;
    {
      const cuuint64_t dims[3] = {(cuuint64_t)d.dstate, (cuuint64_t)d.ngroups,
                                  (cuuint64_t)(d.batch * d.seqlen)};
      const cuuint64_t str[2] = {(cuuint64_t)d.dstate * 2, (cuuint64_t)d.ngroups * d.dstate * 2};
      const cuuint32_t box[3] = {64, 1, (cuuint32_t)ssd::kCorrTile};
      if (!ssd::encode_sw128(&tm_c, true, C, 3, dims, str, box)) return SSD_ERR_CUDA;
    }
    {
      const cuuint64_t row = (cuuint64_t)d.nheads * d.headdim;
      const cuuint64_t dims[3] = {row, (cuuint64_t)d.seqlen, (cuuint64_t)d.batch};
      const cuuint64_t str[2] = {row * es, row * es * (cuuint64_t)d.seqlen};
      const cuuint32_t box[3] = {(cuuint32_t)(128 / es), (cuuint32_t)ssd::kCorrTile, 1};
      if (!ssd::encode_sw128(&tm_y, ob, y, 3, dims, str, box)) return SSD_ERR_CUDA;
    }
    // C tile, staged correction tile, bf16 state block, alignment slack; never more
    // CTAs on an SM than its 512 TMEM columns hold
    size_t smem = 1024 + (size_t)(d.dstate / 64) * ssd::tc::kPanel + (size_t)Pc * es * ssd::kCorrTile +
                  (size_t)Pc * d.dstate * 2;
    const size_t per_sm = 228 * 1024, fit = (size_t)(512 / Pc);
    if (smem <= per_sm / (fit + 1)) smem = per_sm / (fit + 1) + 1;
    if (smem > 227 * 1024) return SSD_ERR_UNSUPPORTED;
    ssd::CorrParams p;
    p.L = d.seqlen;
    p.H = d.nheads;
    p.P = d.headdim;
    p.N = d.dstate;
    p.G = d.ngroups;
    p.Pc = Pc;
    p.out_bf16 = ob;
    p.ntiles = (int)((d.seqlen + ssd::kCorrTile - 1) / ssd::kCorrTile);
    const int64_t units = d.batch * d.nheads * (d.headdim / Pc);
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int64_t per = (int64_t)(per_sm / (smem + 2048)), slots = nsm * (per < 1 ? 1 : per);
    // runs of tiles: short enough for about a dozen items per resident CTA, at least
    // two tiles so the state block is converted no more than every other tile
    int64_t chunk = (units * p.ntiles + 12 * slots - 1) / (12 * slots);
    chunk = chunk < 2 ? 2 : chunk > 8 ? 8 : chunk;
    if (chunk > p.ntiles) chunk = p.ntiles;
    p.chunk = (int)chunk;
    p.items_per_unit = (p.ntiles + p.chunk - 1) / p.chunk;
    if (units * p.items_per_unit > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    p.items = (int)(units * p.items_per_unit);
    p.cs = cs;
    p.h_in = h_in;
    p.status = status;
    const int grid = (int)(p.items < slots ? p.items : slots);
    if (cudaFuncSetAttribute(ssd::cp_correct_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return SSD_ERR_CUDA;
    ssd::cp_correct_tc_kernel<<<grid, 256, smem, st>>>(tm_c, tm_y, p);
    return ssd::launch_rc();
  }
  const size_t smem = sizeof(float) * ((size_t)d.dstate * d.headdim + (size_t)ssd::kCorrTok * d.dstate);
  if (smem > 227 * 1024) return SSD_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(ssd::cp_correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return SSD_ERR_CUDA;
  const int64_t ntile = (d.seqlen + ssd::kCorrTok - 1) / ssd::kCorrTok;
  if (d.batch * d.nheads * ntile > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
  ssd::cp_correct_kernel<<<(unsigned)(d.batch * d.nheads * ntile), 256, smem, st>>>(
      d.seqlen, d.nheads, d.headdim, d.dstate, d.ngroups, d.in_dtype == SSD_BF16,
      d.out_dtype == SSD_BF16, C, cs, h_in, y);
  return ssd::launch_rc();
}
