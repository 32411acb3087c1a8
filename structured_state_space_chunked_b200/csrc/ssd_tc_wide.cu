// ssd_tc_wide.cu -- fused SSD forward on 128-column units (sm_100a tcgen05 + TMEM + TMA).
//
// A work unit is (document, 128 consecutive columns of x viewed as [T, H*P]): two
// heads of P = 64 that share a B/C group, or 128 columns of one head with
// P = 128 or 256.  One persistent CTA walks the unit's tokens in tiles of 128 and
// keeps the running state of all 128 columns in tensor memory.  Per tile j, with
// cs_l the in-tile cumulative log decay of a head ("Transformers are SSMs",
// paperlayer.ai summary, §3.2.2 / §6):
//
//   Z      = C_j B_j^T                    one 128 x 128 product for both heads
//   M_h    = Z o L_h (+ D_h on the diagonal), as bf16 in the other TMEM region
//   Ydiag  = M_h x_j,h                    per head (tensor cores, A from TMEM)
//   Yoff   = C_j Hb_j                     both heads at once, Hb = bf16 state
//   y      = exp(cs_l) Yoff + Ydiag
//   H_j+1  = exp(cs_127) H_j + B_j^T (w o x_j),  w_s = exp(cs_127 - cs_s) delta_s
//
// Sharing C B^T between the heads of a group and running the state update and
// the left factors as N = 128 products is what this kernel adds over the 64-column
// kernel in ssd_tc.cu; it needs N <= 128 (the four 128-column TMEM regions take
// all 512 columns).  C B^T and Ydiag of tile j share region j % 2 and the masks
// go to the other region, so the masks are never written over their own input.
//
// Roles (18 warps): warp 0 owns TMEM and one thread issues the MMAs in tile order;
// one thread of warp 1 runs the loads (x and B/C) as an event loop; warps 2..17 are
// the epilogue, one of whose threads also issues the tile stores of y.  An epilogue warp can only reach the TMEM
// lane quarter warp % 4, so the four warps of a quarter split the columns: warp m
// (0..3) of the quarter takes column block m of Z for the mask, columns
// 32m..32m+31 of the state and outputs, and 16-byte chunks 4(m%2)..4(m%2)+3 of
// panel m/2 in shared memory.
//
// The epilogue is software-pipelined across tiles so that every MMA runs behind
// epilogue work: iteration j builds the masks of tile j, then the scan, w o x and
// state hand-over of tile j+1, then the outputs of tile j.  The tensor pipe runs
// the state update and Yoff of tile j under the masks, Ydiag of tile j under the
// next tile's preparation, and C B^T of tile j+1 under the outputs.  Every
// mbarrier wait is bounded; on expiry the CTA records SSD_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd_internal.h"
#include "tc_common.cuh"

namespace ssd {
namespace {
using namespace tc;

constexpr int kTile = 128;      // tokens per tile
constexpr int kCols = 128;      // columns per unit
constexpr int kEpiWarps = 16;
constexpr int kThreads = 64 + 32 * kEpiWarps;  // 576

struct W {
  static constexpr uint32_t X_BYTES = 2 * kPanel;         // 128 tokens x 128 columns
  static constexpr uint32_t OFF_X = 0;                    // [2] stages
  static constexpr uint32_t OFF_B = 2 * X_BYTES;          // 128 tokens x 128 state (2 panels)
  static constexpr uint32_t OFF_C = OFF_B + 2 * kPanel;
  static constexpr uint32_t OFF_XW = OFF_C + 2 * kPanel;  // w o x, 2 panels
  static constexpr uint32_t OFF_HB = OFF_XW + 2 * kPanel; // bf16 state: 128 rows x 128 columns
  static constexpr uint32_t OFF_Y = OFF_HB + 2 * kPanel;  // y staging tile, 2 panels
  static constexpr uint32_t OFF_V = OFF_Y + 2 * kPanel;   // float[2 head][128]
  static constexpr uint32_t OFF_CT = OFF_V + 1024;        // float[2 head][128]
  static constexpr uint32_t OFF_WS = OFF_CT + 1024;       // float[2 buf][2 head][4], flags at +64
  static constexpr uint32_t OFF_HC = OFF_WS + 128;        // float[2 buf][2 head][4]: A, dt_bias, D
  static constexpr uint32_t OFF_BAR = OFF_HC + 64;
  static constexpr uint32_t OFF_TMEM = OFF_BAR + 256;
  static constexpr uint32_t SMEM = OFF_TMEM + 16;
  // TMEM columns: two 128-column regions that alternate by tile parity p = j % 2
  // (C B^T of tile j and then its Ydiag in region p, its masks in region 1 - p),
  // Yoff, the state
  static constexpr uint32_t COL_R = 0, COL_YO = 256, COL_H = 384;
  static constexpr uint32_t TMEM_COLS = 512;
};
static_assert(W::SMEM <= 232448, "smem budget");

enum Bar {
  X_FULL0 = 0, X_FULL1,    // x tile landed (TMA -> epilogue, MMA)
  X_EMPTY0, X_EMPTY1,      // x stage read by w o x and by Ydiag (MMA commit -> TMA)
  BC_FULL, BC_EMPTY,       // B/C tile landed / read by every MMA of the tile
  CB_DONE,                 // C B^T in Z (MMA -> epilogue)
  M_READY,                 // masks written over Z (epilogue -> MMA)
  XW_READY,                // w o x written (epilogue -> MMA)
  PREP,                    // state decayed in TMEM and Hb written (epilogue -> MMA)
  STATE_DONE,              // state update of the tile done (MMA -> epilogue)
  YO_DONE, YD_DONE,        // Yoff / Ydiag accumulated (MMA -> epilogue; YD_DONE also MMA)
  Y_FREE,                  // Yoff and Ydiag read (epilogue -> MMA)
  TEARDOWN, NBAR
};

struct KParams {
  Geom g;
  const void* dt;
  const float* A;
  const float* D;
  const float* dt_bias;
  const float* init;
  const int32_t* cu;
  __nv_bfloat16* y;
  float* final_states;
  int* status;
  int units;
  int ncb;   // 128-column blocks per token row (H * P / 128)
  int hu;    // heads per unit: 2 (P = 64) or 1
  int hpg;   // heads per B/C group
};

struct Unit {
  int d, col0, h0;
  int64_t start;
  int len, ntiles;
};

__device__ __forceinline__ Unit unit_of(const KParams& k, int u) {
  Unit U;
  const int cb = u % k.ncb;
  U.d = u / k.ncb;
  U.col0 = cb * kCols;
  U.h0 = U.col0 / k.g.P;
  if (k.g.varlen) {
    U.start = k.cu[U.d];
    U.len = (int)((int64_t)k.cu[U.d + 1] - U.start);
  } else {
    U.start = (int64_t)U.d * k.g.seqlen;
    U.len = (int)k.g.seqlen;
  }
  U.ntiles = (U.len + kTile - 1) / kTile;
  return U;
}

struct Cursor {
  int u, jt;
  bool valid;
  Unit U;
};
__device__ __noinline__ int next_unit_with_tiles(const KParams& kp, int u) {
  for (u += gridDim.x; u < kp.units; u += gridDim.x)
    if (unit_of(kp, u).ntiles > 0) return u;
  return -1;
}
__device__ __forceinline__ void cursor_next(const KParams& kp, Cursor& c) {
  if (!c.valid) return;
  if (c.jt + 1 < c.U.ntiles) {
    ++c.jt;
    return;
  }
  c.u = next_unit_with_tiles(kp, c.u);
  c.valid = c.u >= 0;
  c.jt = 0;
  if (c.valid) c.U = unit_of(kp, c.u);
}
__device__ __forceinline__ Cursor cursor_first(const KParams& kp) {
  Cursor c;
  c.u = next_unit_with_tiles(kp, (int)blockIdx.x - (int)gridDim.x);
  c.jt = 0;
  c.valid = c.u >= 0;
  if (c.valid) c.U = unit_of(kp, c.u);
  return c;
}
__device__ __forceinline__ int tile_len(const Cursor& c) { return min(kTile, c.U.len - c.jt * kTile); }
__device__ __forceinline__ int64_t tile_t0(const Cursor& c) {
  return c.U.start + (int64_t)c.jt * kTile;
}
__device__ __noinline__ uint32_t count_tiles(const KParams& kp, int* last_unit) {
  uint32_t n = 0;
  *last_unit = -1;
  for (int u = blockIdx.x; u < kp.units; u += gridDim.x) {
    const Unit U = unit_of(kp, u);
    n += (uint32_t)U.ntiles;
    if (U.ntiles > 0) *last_unit = u;
  }
  return n;
}

__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           int* status) {
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_try(bar, parity)) {
    if ((++n & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > 2000000000ull) {
        *abort_flag = 1;
        set_status(status, SSD_ERR_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* status) {
  return mbar_try(bar, parity) || wait_bar_slow(bar, parity, abort_flag, status);
}

// all 16 epilogue warps
__device__ __forceinline__ void sync_epi() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

// one arrival per warp, after every lane's prior writes
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// The 32 state columns [gc, gc + 32) of unit columns (one head) for state row n:
// offset of element (document d, row n, first column) in [ndocs, H, N, P].
__device__ __forceinline__ int64_t state_off(const KParams& kp, int d, int gc, int n) {
  const int h = gc / kp.g.P, p = gc % kp.g.P;
  return (((int64_t)d * kp.g.H + h) * kp.g.N + n) * kp.g.P + p;
}

// 32 state columns of TMEM row n -> final_states
__device__ __noinline__ void state_to_final(const KParams& kp, uint32_t th, int d, int gc, int n) {
  float hv[32];
  tc_ld32(th, hv);
  tc_wait_ld();
  if (!kp.final_states || n >= kp.g.N) return;
  float* dst = kp.final_states + state_off(kp, d, gc, n);
#pragma unroll
  for (int c = 0; c < 32; c += 4)
    *reinterpret_cast<float4*>(dst + c) = make_float4(hv[c], hv[c + 1], hv[c + 2], hv[c + 3]);
}

// Entry into a unit: the initial state (or zero) of row n, 32 columns, goes to Hb
// as bf16 (4 chunks of panel `hb_panel`) and, decayed, into TMEM.
__device__ __noinline__ void enter_state(const KParams& kp, uint32_t th, uint32_t hb_panel,
                                         uint32_t chunk0, int d, int gc, int n, float decay) {
  const float* src = (kp.init && n < kp.g.N) ? kp.init + state_off(kp, d, gc, n) : nullptr;
  float hv[32];
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    const float4 f = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0, 0, 0, 0);
    hv[c] = f.x;
    hv[c + 1] = f.y;
    hv[c + 2] = f.z;
    hv[c + 3] = f.w;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    st_shared_v4(hb_panel + swz((uint32_t)n, chunk0 + c), pack_bf16(hv[8 * c], hv[8 * c + 1]),
                 pack_bf16(hv[8 * c + 2], hv[8 * c + 3]), pack_bf16(hv[8 * c + 4], hv[8 * c + 5]),
                 pack_bf16(hv[8 * c + 6], hv[8 * c + 7]));
#pragma unroll
  for (int c = 0; c < 32; ++c) hv[c] *= decay;
  tc_st32(th, hv);
}

// Documents without tokens: final state = initial state (or zero).  Spread over
// the 512 epilogue threads.
__device__ __noinline__ void empty_units_final(const KParams& kp, int tid) {
  if (!kp.final_states) return;
  for (int u = blockIdx.x; u < kp.units; u += gridDim.x) {
    const Unit U = unit_of(kp, u);
    if (U.ntiles != 0) continue;
    for (int e = tid; e < kp.g.N * kCols; e += 32 * kEpiWarps) {
      const int n = e / kCols, c = e % kCols;
      const int64_t off = state_off(kp, U.d, U.col0 + c, n);
      kp.final_states[off] = kp.init ? kp.init[off] : 0.f;
    }
  }
}

// Off-diagonal column block (all columns before the row's own 32-block): with
// b the last token of the block, exp(cs_r - cs_b) exp(cs_b - cs_s) = exp(cs_r - cs_s)
// and both factors are <= 1; vcol[s] = exp(cs_b - cs_s) delta_s.  16 columns in,
// 8 bf16 pairs out.
__device__ __forceinline__ void mask_off16(const float* zv, float u, const float* vcol,
                                           uint32_t* pk) {
  const uint64_t uu = f2_pack(u, u);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float4 vv = *reinterpret_cast<const float4*>(vcol + 2 * i);
    const uint64_t a = f2_mul(f2_pack(zv[2 * i], zv[2 * i + 1]), f2_mul(uu, f2_pack(vv.x, vv.y)));
    const uint64_t b =
        f2_mul(f2_pack(zv[2 * i + 2], zv[2 * i + 3]), f2_mul(uu, f2_pack(vv.z, vv.w)));
    pk[i] = f2_to_bf16x2(a);
    pk[i + 1] = f2_to_bf16x2(b);
  }
}
// Diagonal 32 x 32 block (rows = this warp's lanes), columns j0..j0+15 of it:
// M[r, s] = Z exp(cs_r - cs_s) delta_s for s <= r, written 2^(cs_r - ct_s) with
// ct_s = cs_s - log2(delta_s) (+inf when delta_s = 0); D on the diagonal.
__device__ __forceinline__ void mask_diag16(const float* zv, float cs, const float* ctcol, int j0,
                                            int lane, float Dh, uint32_t* pk) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float4 t = *reinterpret_cast<const float4*>(ctcol + 2 * i);
    const float ctj[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int a = 2 * (i + k), j = j0 + a;
      float m0 = zv[a] * ex2(cs - ctj[2 * k]);
      float m1 = zv[a + 1] * ex2(cs - ctj[2 * k + 1]);
      m0 = j == lane ? m0 + Dh : m0;
      m1 = j + 1 == lane ? m1 + Dh : m1;
      m0 = j <= lane ? m0 : 0.f;
      m1 = j + 1 <= lane ? m1 : 0.f;
      pk[i + k] = pack_bf16(m0, m1);
    }
  }
}

// The copy thread: two in-order streams over the CTA's tiles -- x loads (two
// stages, up to two tiles ahead) and B/C loads (one buffer) -- polled without
// blocking so that whichever is ready goes.  With each x tile it also writes the
// per-head constants of the tile's unit (A, dt_bias, D) to slot (tile % 2); they
// are visible to whoever waits for that tile's x.  Kept out of line so that its
// cursors do not weigh on the register allocation of the epilogue.
__device__ __noinline__ void copy_loop(const CUtensorMap* tm_x, const CUtensorMap* tm_b,
                                       const CUtensorMap* tm_c, const KParams& kp, uint32_t sbase,
                                       volatile int* abort_flag) {
  auto bar = [&](int i) { return sbase + W::OFF_BAR + 8u * (uint32_t)i; };
  Cursor cx = cursor_first(kp), cb = cx;
  uint32_t nx = 0, nbc = 0;
  int hc_unit = -1;
  float hc[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  uint64_t t_idle = 0;
  uint32_t idle = 0;
  while ((cx.valid || cb.valid) && !*abort_flag) {
    bool did = false;
    if (cb.valid && (nbc == 0 || mbar_test(bar(BC_EMPTY), (nbc - 1) & 1))) {
      const int t0 = (int)tile_t0(cb);
      const int grp = cb.U.h0 / kp.hpg;
      mbar_expect_tx(bar(BC_FULL), 4 * kPanel);
      tma_3d(sbase + W::OFF_B, tm_b, bar(BC_FULL), 0, grp, t0);
      tma_3d(sbase + W::OFF_B + kPanel, tm_b, bar(BC_FULL), 64, grp, t0);
      tma_3d(sbase + W::OFF_C, tm_c, bar(BC_FULL), 0, grp, t0);
      tma_3d(sbase + W::OFF_C + kPanel, tm_c, bar(BC_FULL), 64, grp, t0);
      cursor_next(kp, cb);
      ++nbc;
      did = true;
    }
    if (cx.valid && (nx < 2 || mbar_test(bar(X_EMPTY0 + (nx & 1)), ((nx >> 1) - 1) & 1))) {
      const uint32_t s = nx & 1u;
      if (cx.u != hc_unit) {
        hc_unit = cx.u;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = min(cx.U.h0 + hh, kp.g.H - 1);
          hc[3 * hh] = kp.A[h];
          hc[3 * hh + 1] = kp.dt_bias ? kp.dt_bias[h] : 0.f;
          hc[3 * hh + 2] = kp.D ? kp.D[h] : 0.f;
        }
      }
      const uint32_t hs = sbase + W::OFF_HC + 32u * s;
      st_shared_v4(hs, __float_as_uint(hc[0]), __float_as_uint(hc[1]), __float_as_uint(hc[2]), 0u);
      st_shared_v4(hs + 16, __float_as_uint(hc[3]), __float_as_uint(hc[4]), __float_as_uint(hc[5]), 0u);
      const int t0 = (int)tile_t0(cx);
      const uint32_t xs = sbase + W::OFF_X + s * W::X_BYTES;
      mbar_expect_tx(bar(X_FULL0 + s), W::X_BYTES);
      tma_2d(xs, tm_x, bar(X_FULL0 + s), cx.U.col0, t0);
      tma_2d(xs + kPanel, tm_x, bar(X_FULL0 + s), cx.U.col0 + 64, t0);
      cursor_next(kp, cx);
      ++nx;
      did = true;
    }
    if (did) {
      idle = 0;
      t_idle = 0;
    } else if ((++idle & 15u) != 0) {
      __nanosleep(32);
    } else {
      const uint64_t now = globaltimer();
      if (t_idle == 0) {
        t_idle = now;
      } else if (now - t_idle > 2000000000ull) {
        *abort_flag = 1;
        set_status(kp.status, SSD_ERR_TIMEOUT);
        break;
      }
    }
  }
  // drain: every issued load has landed before the CTA exits (already true on the
  // normal path; bounded to ~0.1 s otherwise)
  const uint64_t t0 = globaltimer();
  for (uint32_t i = nx >= 2 ? nx - 2 : 0; i < nx; ++i) {
    while (!mbar_try(bar(X_FULL0 + (i & 1)), (i >> 1) & 1) && globaltimer() - t0 < 100000000ull) {
    }
  }
  if (nbc > 0)
    while (!mbar_try(bar(BC_FULL), (nbc - 1) & 1) && globaltimer() - t0 < 100000000ull) {
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    ssd_tc_wide(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                const __grid_constant__ KParams kp) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = su32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* v_all = reinterpret_cast<float*>(smem + W::OFF_V);
  float* ct_all = reinterpret_cast<float*>(smem + W::OFF_CT);
  float* ws_all = reinterpret_cast<float*>(smem + W::OFF_WS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + W::OFF_WS + 64);
  int* bad_flag = reinterpret_cast<int*>(smem + W::OFF_WS + 68);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + W::OFF_TMEM);
  auto bar = [&](int i) { return sbase + W::OFF_BAR + 8u * (uint32_t)i; };
  const Geom& g = kp.g;

  // ---- set-up: alignment check, cu_seqlens check, barriers, TMEM ----------------
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *bad_flag = (sbase & 1023u) != 0 ? 2 : 0;
  }
  __syncthreads();
  if (g.varlen) {
    int bad = 0;
    for (int d = threadIdx.x; d <= g.ndocs; d += kThreads) {
      const int64_t v = kp.cu[d];
      if (d == 0 && v != 0) bad = 1;
      if (d == g.ndocs && v != g.tokens) bad = 1;
      if (d > 0 && v < (int64_t)kp.cu[d - 1]) bad = 1;
    }
    if (bad) atomicOr(bad_flag, 1);
  }
  __syncthreads();
  if (*bad_flag) {
    if (threadIdx.x == 0)
      set_status(kp.status, (*bad_flag & 1) ? SSD_ERR_BAD_SEQLENS : SSD_ERR_INVALID_ARG);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      const bool per_warp = i == M_READY || i == XW_READY || i == PREP || i == Y_FREE;
      mbar_init(bar(i), per_warp ? kEpiWarps : 1);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(tmem_slot)),
                 "r"(W::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int last_unit = -1;
  const uint32_t ntiles = count_tiles(kp, &last_unit);

  if (warp == 1) {
    // ============================ copies (event loop) =============================
    if (lane == 0) copy_loop(&tm_x, &tm_b, &tm_c, kp, sbase, abort_flag);
  } else if (warp == 0) {
    // ================================ MMA issuer =================================
    if (lane == 0) {
      constexpr uint32_t ID_CB = idesc(128, 128, 0, 0);   // Z = C B^T, both K-major
      constexpr uint32_t ID_ST = idesc(128, 128, 1, 1);   // H += B^T XW, both MN-major
      constexpr uint32_t ID_YO = idesc(128, 128, 0, 1);   // Yoff = C Hb, Hb MN-major
      constexpr uint32_t ID_YD2 = idesc(128, 64, 0, 1);   // Ydiag per head of 64
      constexpr uint32_t ID_YD1 = idesc(128, 128, 0, 1);  // Ydiag of one 128-column head
      const uint64_t dC = sdesc(sbase + W::OFF_C, 16, 1024);
      const uint64_t dB = sdesc(sbase + W::OFF_B, 16, 1024);
      const uint64_t dBm = sdesc(sbase + W::OFF_B, kPanel, 1024);
      const uint64_t dXW = sdesc(sbase + W::OFF_XW, kPanel, 1024);
      const uint64_t dHb = sdesc(sbase + W::OFF_HB, kPanel, 1024);
      bool ok = true;
      for (uint32_t j = 0; j < ntiles && ok; ++j) {
        const uint32_t s = j & 1u, ph = j & 1u;
        // ---- Z = C_j B_j^T into region p (after Ydiag of the previous tile read its
        // masks from there) ----
        ok = wait_bar(bar(BC_FULL), ph, abort_flag, kp.status);
        if (ok && j > 0) ok = wait_bar(bar(YD_DONE), ph ^ 1, abort_flag, kp.status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = ((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
          tc_mma(tmem + W::COL_R + 128 * ph, dC + off, dB + off, ID_CB, kk > 0);
        }
        tc_commit(bar(CB_DONE));
        // ---- state update and left factors ----
        ok = wait_bar(bar(XW_READY), ph, abort_flag, kp.status) &&
             wait_bar(bar(PREP), ph, abort_flag, kp.status) &&
             (j == 0 || wait_bar(bar(Y_FREE), ph ^ 1, abort_flag, kp.status));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk)
          tc_mma(tmem + W::COL_H, dBm + ((kk * 2048) >> 4), dXW + ((kk * 2048) >> 4), ID_ST, 1);
        tc_commit(bar(STATE_DONE));
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = ((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
          tc_mma(tmem + W::COL_YO, dC + off, dHb + ((kk * 2048) >> 4), ID_YO, kk > 0);
        }
        tc_commit(bar(YO_DONE));
        tc_commit(bar(BC_EMPTY));
        // ---- Ydiag = M x_j per head, M from TMEM ----
        ok = wait_bar(bar(M_READY), ph, abort_flag, kp.status) &&
             wait_bar(bar(X_FULL0 + s), (j >> 1) & 1, abort_flag, kp.status);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dX = sdesc(sbase + W::OFF_X + s * W::X_BYTES, kPanel, 1024);
        // masks in region 1 - p, Ydiag over the spent C B^T in region p
        const uint32_t rm = tmem + W::COL_R + 128 * (ph ^ 1), ry = tmem + W::COL_R + 128 * ph;
        if (kp.hu == 2) {
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll 1
            for (int kk = 0; kk < 8; ++kk)
              tc_mma_ts(ry + 64 * hh, rm + 32 * (kk >> 1) + 16 * hh + 8 * (kk & 1),
                        dX + ((hh * kPanel + kk * 2048) >> 4), ID_YD2, kk > 0);
        } else {
#pragma unroll 1
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ts(ry, rm + 32 * (kk >> 1) + 8 * (kk & 1), dX + ((kk * 2048) >> 4), ID_YD1,
                      kk > 0);
        }
        tc_commit(bar(YD_DONE));
        tc_commit(bar(X_EMPTY0 + s));
      }
      // every MMA this thread issued has completed once TEARDOWN fires
      tc_commit(bar(TEARDOWN));
      // bounded by time only: TMEM is freed below, so no MMA may still run then
      if (!wait_drain(bar(TEARDOWN), 0, 2000000000ull)) set_status(kp.status, SSD_ERR_TIMEOUT);
    }
  } else {
    // ================================ epilogue ==================================
    const int q = warp & 3;            // TMEM lane quarter
    const int m = (warp - 2) >> 2;     // column share within the quarter
    const int r = q * 32 + lane;       // tile row (token) == TMEM lane == state row
    const int tid = (warp - 2) * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int pn = m >> 1;             // shared-memory panel of this warp's columns
    const uint32_t ch0 = 4u * (uint32_t)(m & 1);  // first 16-byte chunk in the panel
    const int hu = kp.hu;
    const int hw = hu == 2 ? pn : 0;   // head (within the unit) of this warp's columns
    const float LOG2E = 1.4426950408889634f;
    empty_units_final(kp, tid);

    // raw bf16 dt of a tile for this thread's row, both heads in one word (lo, hi):
    // one aligned 32-bit load for a head pair (h0 and H are even), else 16 bits.
    // Nothing touches the register until the scan uses it, so the load latency
    // stays off this thread until then.
    auto load_dt = [&](const Cursor& c) -> uint32_t {
      if (!c.valid || r >= tile_len(c)) return 0u;
      const __nv_bfloat16* p =
          reinterpret_cast<const __nv_bfloat16*>(kp.dt) + (tile_t0(c) + r) * g.H + c.U.h0;
      return hu == 2 ? ld_global_u32(p) : ld_global_u16(p);
    };
    // per-head scan totals of 32-row blocks of tile buffer b -> the cumulative
    // log2 decay at the end of blocks 0..3
    auto block_ends = [&](uint32_t b, int hh) -> float4 {
      const float4 t = *reinterpret_cast<const float4*>(ws_all + 8 * b + 4 * hh);
      const float e0 = t.x, e1 = e0 + t.y, e2 = e1 + t.z;
      return make_float4(e0, e1, e2, e2 + t.w);
    };

    // Live across iterations: cs of both heads (mask), w and exp(cs) of this
    // warp's head (w o x, outputs).  Everything else is recomputed from shared memory.
    float cs[2] = {0.f, 0.f}, wr = 0.f, el = 0.f;
    // E1 of a tile: one scan per head; v and ct columns to shared memory, block
    // totals to ws buffer b.  The barrier inside also orders every warp's masks of
    // the previous tile (which read v and ct) before the new values are written;
    // the barrier at the top of the tile loop publishes them.
    auto stage1 = [&](const Cursor& c, uint32_t dtw, uint32_t b) {
      const int len = tile_len(c);
      float dl[2] = {0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (hh >= hu) break;
        float la = 0.f;
        if (r < len) {
          // A and dt_bias of the head, from the slot written with this tile's x
          const uint4 hc = ld_shared_v4(sbase + W::OFF_HC + 32u * b + 16u * hh);
          const float dtv = __uint_as_float((hh ? dtw >> 16 : dtw & 0xffffu) << 16);
          dl[hh] = softplus_f(dtv + __uint_as_float(hc.y));
          la = dl[hh] * __uint_as_float(hc.x) * LOG2E;
        }
        float x = la;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float t = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += t;
        }
        if (m == 0 && lane == 31) ws_all[8 * b + 4 * hh + q] = x;
        cs[hh] = x;
      }
      // the previous tile store has read the staging tile before anyone passes here
      if (tid == 0) bulk_wait_read0();
      sync_epi();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (hh >= hu) break;
        const float4 e = block_ends(b, hh);
        const float base = q == 0 ? 0.f : q == 1 ? e.x : q == 2 ? e.y : e.z;
        const float cend = q == 0 ? e.x : q == 1 ? e.y : q == 2 ? e.z : e.w;
        const float x = cs[hh] + base;
        cs[hh] = x;
        if (m == 0) {
          v_all[128 * hh + r] = ex2(cend - x) * dl[hh];
          ct_all[128 * hh + r] =
              dl[hh] > 0.f ? x - __log2f(dl[hh]) : __int_as_float(0x7f800000);
        }
        if (hh == hw) {
          wr = ex2(e.w - x) * dl[hh];
          el = ex2(x);
        }
      }
    };
    // E4: XW = w o x of the tile in x stage s (MN-major B operand of the state update)
    auto stage4 = [&](uint32_t s) {
      const uint64_t ww = f2_pack(wr, wr);
      const uint32_t xp = sbase + W::OFF_X + s * W::X_BYTES + pn * kPanel;
      const uint32_t xwp = sbase + W::OFF_XW + pn * kPanel;
#pragma unroll
      for (uint32_t c = 0; c < 4; ++c) {
        const uint32_t a = swz((uint32_t)r, ch0 + c);
        const uint4 xv = ld_shared_v4(xp + a);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
        const float2 f0 = __bfloat1622float2(p2[0]), f1 = __bfloat1622float2(p2[1]);
        const float2 f2 = __bfloat1622float2(p2[2]), f3 = __bfloat1622float2(p2[3]);
        st_shared_v4(xwp + a, f2_to_bf16x2(f2_mul(ww, f2_pack(f0.x, f0.y))),
                     f2_to_bf16x2(f2_mul(ww, f2_pack(f1.x, f1.y))),
                     f2_to_bf16x2(f2_mul(ww, f2_pack(f2.x, f2.y))),
                     f2_to_bf16x2(f2_mul(ww, f2_pack(f3.x, f3.y))));
      }
      fence_async_smem();
      warp_arrive(bar(XW_READY), lane);
    };
    // E3: the state entering tile c (H in TMEM is the state after the previous
    // tile's update, or the previous unit's final state when c starts a unit)
    auto stage3 = [&](const Cursor& c, uint32_t b, int prev_u) {
      tc_fence_after();
      const float decay = ex2(block_ends(b, hw).w);
      const uint32_t th = tmem + lane_off + W::COL_H + 32 * m;
      const uint32_t hbp = sbase + W::OFF_HB + pn * kPanel;
      if (c.jt == 0) {
        if (prev_u >= 0) {
          const Unit P = unit_of(kp, prev_u);
          state_to_final(kp, th, P.d, P.col0 + 32 * m, r);
        }
        enter_state(kp, th, hbp, ch0, c.U.d, c.U.col0 + 32 * m, r, decay);
      } else {
        const uint64_t dd = f2_pack(decay, decay);
        float hv[16], hn[16];
        tc_ld16(th, hv);
        tc_wait_ld();
#pragma unroll 1
        for (uint32_t hf = 0; hf < 2; ++hf) {
          if (hf == 0) tc_ld16(th + 16, hn);
#pragma unroll
          for (uint32_t cq = 0; cq < 2; ++cq)
            st_shared_v4(hbp + swz((uint32_t)r, ch0 + 2 * hf + cq), pack_bf16(hv[8 * cq], hv[8 * cq + 1]),
                         pack_bf16(hv[8 * cq + 2], hv[8 * cq + 3]),
                         pack_bf16(hv[8 * cq + 4], hv[8 * cq + 5]),
                         pack_bf16(hv[8 * cq + 6], hv[8 * cq + 7]));
          uint32_t o[16];
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const uint64_t v2 = f2_mul(dd, f2_pack(hv[k], hv[k + 1]));
            o[k] = (uint32_t)v2;
            o[k + 1] = (uint32_t)(v2 >> 32);
          }
          tc_st16(th + 16 * hf, o);
          if (hf == 0) {
            tc_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) hv[k] = hn[k];
          }
        }
      }
      tc_wait_st();
      fence_async_smem();
      tc_fence_before();
      warp_arrive(bar(PREP), lane);
    };

    bool ok = true;
    Cursor cur = cursor_first(kp);
    uint32_t dt_next = 0;  // raw dt of the tile after cur
    // ---- prologue: E1, E4, E3 of the first tile ----
    if (cur.valid) {
      const uint32_t dt0 = load_dt(cur);
      {
        Cursor nx = cur;
        cursor_next(kp, nx);
        dt_next = load_dt(nx);
      }
      ok = wait_bar(bar(X_FULL0), 0, abort_flag, kp.status);  // also publishes the head constants
      if (ok) {
        stage1(cur, dt0, 0);
        stage4(0);
        stage3(cur, 0, -1);
      }
    }

    uint32_t j = 0;
    for (; cur.valid && ok; ++j) {
      const uint32_t ph = j & 1u, b = j & 1u;

      // ---- E2 of tile j: decay masks from C B^T ----
      // (the barrier makes every warp's v / ct columns of tile j visible, and orders
      // every warp's reads of Ydiag of tile j-1, in the region the masks now take)
      sync_epi();
      ok = wait_bar(bar(CB_DONE), ph, abort_flag, kp.status);
      if (!ok) break;
      tc_fence_after();
      {
        // Column block cc of Z (32 columns, region p) becomes 16 packed columns per
        // head at 32cc + 16hh of region 1 - p.  The four warps of the quarter split
        // every block that is not all zero: warp m takes its columns 8m..8m+7
        // (pairs at 32cc + 16hh + 4m), so each carries a quarter of the diagonal block.
        const uint32_t zin = tmem + lane_off + W::COL_R + 128u * ph;
        const uint32_t zout = tmem + lane_off + W::COL_R + 128u * (ph ^ 1u);
        if (m > q) {
          // block m lies above the diagonal for these rows: all zero
          uint32_t zero[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) zero[i] = 0u;
          tc_st16(zout + 32 * m, zero);
          if (hu == 2) tc_st16(zout + 32 * m + 16, zero);
        }
#pragma unroll 1
        for (int cc = 0; cc <= q; ++cc) {
          float za[8];
          tc_ld8(zin + 32 * cc + 8 * m, za);
          tc_wait_ld();
          if (cc < q) {
            // off-diagonal: exp(cs_r - cs_end(cc)) v_s
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (hh >= hu) break;
              // cumulative log2 decay at the end of block cc: sum of the block totals
              const uint4 t4 = ld_shared_v4(sbase + W::OFF_WS + 32u * b + 16u * hh);
              const float w0 = __uint_as_float(t4.x), w1 = __uint_as_float(t4.y);
              const float be = cc == 0 ? w0 : cc == 1 ? w0 + w1 : w0 + w1 + __uint_as_float(t4.z);
              const float u = ex2(cs[hh] - be);
              const uint64_t uu = f2_pack(u, u);
              const uint32_t vc = sbase + W::OFF_V + 4u * (128 * hh + 32 * cc + 8 * m);
              const uint4 va = ld_shared_v4(vc), vb4 = ld_shared_v4(vc + 16);
              const float vv[8] = {__uint_as_float(va.x), __uint_as_float(va.y), __uint_as_float(va.z),
                                   __uint_as_float(va.w), __uint_as_float(vb4.x), __uint_as_float(vb4.y),
                                   __uint_as_float(vb4.z), __uint_as_float(vb4.w)};
              uint32_t pk[4];
#pragma unroll
              for (int i = 0; i < 4; ++i)
                pk[i] = f2_to_bf16x2(f2_mul(f2_pack(za[2 * i], za[2 * i + 1]),
                                            f2_mul(uu, f2_pack(vv[2 * i], vv[2 * i + 1]))));
              tc_st4(zout + 32 * cc + 16 * hh + 4 * m, pk);
            }
          } else {
            // diagonal block, columns j = 8m + i: 2^(cs_r - ct_s) for j <= lane, D at j == lane
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (hh >= hu) break;
              const uint32_t cp = sbase + W::OFF_CT + 4u * (128 * hh + 32 * q + 8 * m);
              const uint4 ca = ld_shared_v4(cp), cb4 = ld_shared_v4(cp + 16);
              const float ctv[8] = {__uint_as_float(ca.x), __uint_as_float(ca.y), __uint_as_float(ca.z),
                                    __uint_as_float(ca.w), __uint_as_float(cb4.x), __uint_as_float(cb4.y),
                                    __uint_as_float(cb4.z), __uint_as_float(cb4.w)};
              const float Dh = __uint_as_float(ld_shared_v4(sbase + W::OFF_HC + 32u * b + 16u * hh).z);
              const float csr = cs[hh];
              uint32_t pk[4];
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                const int j = 8 * m + i;
                float m0 = za[i] * ex2(csr - ctv[i]);
                float m1 = za[i + 1] * ex2(csr - ctv[i + 1]);
                m0 = j == lane ? m0 + Dh : m0;
                m1 = j + 1 == lane ? m1 + Dh : m1;
                m0 = j <= lane ? m0 : 0.f;
                m1 = j + 1 <= lane ? m1 : 0.f;
                pk[i >> 1] = pack_bf16(m0, m1);
              }
              tc_st4(zout + 32 * q + 16 * hh + 4 * m, pk);
            }
          }
        }
      }
      tc_wait_st();
      tc_fence_before();
      warp_arrive(bar(M_READY), lane);

      // ---- E1, E4, E3 of tile j+1, while the tensor cores run Ydiag of tile j ----
      const float el_cur = el;
      Cursor nxt = cur;
      cursor_next(kp, nxt);
      uint32_t dt_next2 = 0;
      {
        Cursor n2 = nxt;
        cursor_next(kp, n2);
        dt_next2 = load_dt(n2);  // consumed one iteration later
      }
      if (nxt.valid) {
        // x of tile j+1 (with its head constants) has landed
        ok = wait_bar(bar(X_FULL0 + (b ^ 1u)), ((j + 1) >> 1) & 1, abort_flag, kp.status);
        if (!ok) break;
        stage1(nxt, dt_next, b ^ 1u);
        // XW and the state may be overwritten once the state update of tile j is done
        ok = wait_bar(bar(STATE_DONE), ph, abort_flag, kp.status);
        if (!ok) break;
        stage4(b ^ 1u);
        // Hb may be overwritten once Yoff of tile j has read it
        ok = wait_bar(bar(YO_DONE), ph, abort_flag, kp.status);
        if (!ok) break;
        stage3(nxt, b ^ 1u, nxt.jt == 0 ? cur.u : -1);
      }
      dt_next = dt_next2;

      // ---- E5 of tile j: y = exp(cs) Yoff + Ydiag into the staging tile ----
      if (!nxt.valid) {
        // no E1 barrier this iteration: wait for the previous tile store here
        if (tid == 0) bulk_wait_read0();
        sync_epi();
      }
      ok = wait_bar(bar(YO_DONE), ph, abort_flag, kp.status) &&
           wait_bar(bar(YD_DONE), ph, abort_flag, kp.status);
      if (!ok) break;
      tc_fence_after();
      {
        float yo[32], yd[32];
        tc_ld16(tmem + lane_off + W::COL_YO + 32 * m, yo);
        tc_ld16(tmem + lane_off + W::COL_YO + 32 * m + 16, yo + 16);
        tc_ld16(tmem + lane_off + W::COL_R + 128 * ph + 32 * m, yd);
        tc_ld16(tmem + lane_off + W::COL_R + 128 * ph + 32 * m + 16, yd + 16);
        tc_wait_ld();
        tc_fence_before();
        warp_arrive(bar(Y_FREE), lane);
        const uint64_t ee = f2_pack(el_cur, el_cur);
        const uint32_t sp = sbase + W::OFF_Y + pn * kPanel;
#pragma unroll
        for (uint32_t c = 0; c < 4; ++c) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 8 * c + 2 * i;
            o[i] = f2_to_bf16x2(f2_fma(ee, f2_pack(yo[k], yo[k + 1]), f2_pack(yd[k], yd[k + 1])));
          }
          st_shared_v4(sp + swz((uint32_t)r, ch0 + c), o[0], o[1], o[2], o[3]);
        }
      }
      const int len = tile_len(cur);
      fence_async_smem();
      sync_epi();
      if (len == kTile) {
        // whole tile: one tensor store per panel, read out before the next E1 barrier
        if (tid == 0) {
          const int t0 = (int)tile_t0(cur);
          tma_store_2d(&tm_y, sbase + W::OFF_Y, cur.U.col0, t0);
          tma_store_2d(&tm_y, sbase + W::OFF_Y + kPanel, cur.U.col0 + 64, t0);
          bulk_commit();
        }
      } else {
        // a partial tile (end of a document): rows past its end belong to the next
        // document, so it is stored row by row
        __nv_bfloat16* ybase = kp.y + cur.U.col0;
        const int64_t t0 = tile_t0(cur);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = tid + 512 * i, row = e >> 4, c16 = e & 15;
          if (row < len) {
            const uint4 v = ld_shared_v4(sbase + W::OFF_Y + (uint32_t)(c16 >> 3) * kPanel +
                                         swz((uint32_t)row, (uint32_t)(c16 & 7)));
            *reinterpret_cast<uint4*>(ybase + (t0 + row) * (int64_t)g.H * g.P + c16 * 8) = v;
          }
        }
      }
      cur = nxt;
    }
    if (tid == 0) bulk_wait0();  // every tile store complete before the CTA exits
    // the last unit's final state (after the last tile's state update)
    if (ok && ntiles > 0 && last_unit >= 0) {
      ok = wait_bar(bar(STATE_DONE), (ntiles - 1) & 1, abort_flag, kp.status);
      if (ok) {
        tc_fence_after();
        const Unit L = unit_of(kp, last_unit);
        state_to_final(kp, tmem + lane_off + W::COL_H + 32 * m, L.d, L.col0 + 32 * m, r);
      }
    }
  }

  // ---- teardown ----
  __syncwarp();  // lanes 1..31 of the MMA and copy warps wait for lane 0
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(W::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace

// 128-column units apply when every unit's heads share one B/C group and the
// state fits the 128 TMEM lanes.
bool tc_wide_supported(const Geom& g) {
  if (g.N > 128) return false;
  if (g.P % 128 == 0) return g.P <= 256;
  return g.P == 64 && (g.H / g.G) % 2 == 0;
}

int tc_wide_units(const Geom& g) { return g.ndocs * (g.H * g.P / kCols); }

cudaError_t tc_wide_forward(const Geom& g, const Args& a, int* status, cudaStream_t stream,
                            int num_sms) {
  CUtensorMap tx, tb, tc, ty;
  const cuuint64_t T = (cuuint64_t)g.tokens;
  {
    cuuint64_t dims[2] = {(cuuint64_t)g.H * g.P, T};
    cuuint64_t str[1] = {(cuuint64_t)g.H * g.P * 2};
    cuuint32_t box[2] = {64, kTile};
    if (!tc::encode_bf16_sw128(&tx, a.x, 2, dims, str, box)) return cudaErrorInvalidValue;
    if (!tc::encode_bf16_sw128(&ty, a.y, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)g.N, (cuuint64_t)g.G, T};
    cuuint64_t str[2] = {(cuuint64_t)g.N * 2, (cuuint64_t)g.G * g.N * 2};
    cuuint32_t box[3] = {64, 1, kTile};
    if (!tc::encode_bf16_sw128(&tb, a.B, 3, dims, str, box)) return cudaErrorInvalidValue;
    if (!tc::encode_bf16_sw128(&tc, a.C, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  KParams kp;
  kp.g = g;
  kp.dt = a.dt;
  kp.A = a.A;
  kp.D = a.D;
  kp.dt_bias = a.dt_bias;
  kp.init = a.init;
  kp.cu = a.cu;
  kp.y = reinterpret_cast<__nv_bfloat16*>(a.y);
  kp.final_states = a.final_states;
  kp.status = status;
  kp.ncb = g.H * g.P / kCols;
  kp.units = tc_wide_units(g);
  kp.hu = g.P == 64 ? 2 : 1;
  kp.hpg = g.H / g.G;
  const int grid = kp.units < num_sms ? kp.units : num_sms;
  cudaError_t e = cudaFuncSetAttribute(ssd_tc_wide, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)W::SMEM);
  if (e != cudaSuccess) return e;
  ssd_tc_wide<<<grid, kThreads, W::SMEM, stream>>>(tx, tb, tc, ty, kp);
  return cudaGetLastError();
}

}  // namespace ssd
