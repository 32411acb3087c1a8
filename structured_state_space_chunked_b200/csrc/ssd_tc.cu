// ssd_tc.cu -- fused SSD forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel.  A work unit is (document, head, 64-wide slice of the
// head dimension P); a CTA walks the unit's tokens in tiles of 128 and keeps the
// running SSM state of the slice in tensor memory the whole way, so chunk states
// never touch HBM.  Per tile j (tokens t0..t0+127 of one document):
//
//   cs_l   = sum_{k<=l} delta_k A            (in-tile cumulative log decay, §3.2.2)
//   Z      = C_j B_j^T                       (128 x 128, tensor cores)
//   M[l,s] = Z[l,s] exp(cs_l - cs_s) delta_s for s <= l, 0 above; M[l,l] += D
//                                            (the masked quadratic form of the
//                                             diagonal block, §6.1 / §5.1)
//   Ydiag  = M x_j                           (tensor cores)
//   Yoff   = C_j H_j                         (left factors, §6.2; H_j = state
//                                             entering the tile, bf16 copy)
//   y      = exp(cs_l) Yoff + Ydiag
//   H_{j+1}= exp(cs_127) H_j + B_j^T (w o x_j),  w_s = exp(cs_127 - cs_s) delta_s
//                                            (right factors + the scalar scan
//                                             across chunks, §6.2), accumulated
//                                             by the tensor cores onto the
//                                             decayed state in TMEM.
//
// A chunk of Q = 128 or 256 tokens ("Transformers are SSMs", paperlayer.ai
// summary, §6) is processed as Q/128 such tiles: for Q = 256 the strictly lower
// 128 x 128 block of the chunk's quadratic form goes through the same rank-N
// factorisation the decomposition uses between chunks (the mask L restricted to
// a strictly lower block is rank one, §3.2.2), which equals the quadratic form
// up to rounding.
//
// Roles: warp 0 owns TMEM and one of its threads issues every tcgen05.mma, warp 1
// issues the TMA loads (x/B/C tiles, double-buffered when they fit), and two
// epilogue groups of four warps (2..5 and 6..9) take alternate tiles end to end:
// cumulative decay, w o x, the decay-masked operand M (written over C B^T in
// TMEM, as bf16), the state hand-over and the outputs.  This kernel takes 64-wide
// column units; ssd_tc_wide.cu takes 128-wide ones where the shape allows.  Every
// mbarrier wait is bounded: on expiry the CTA records SSD_ERR_TIMEOUT in the status
// word and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd_ext.h"
#include "ssd_internal.h"
#include "tc_common.cuh"

namespace ssd {
namespace {
using namespace tc;

constexpr int kTile = 128;          // tokens per tile
constexpr int kPT = 64;             // head-dim columns per unit
constexpr int kThreads = 320;       // 10 warps: MMA, TMA, two epilogue groups of 4

template <int NT>
struct Cfg {
  static constexpr int NPAD = 128 * NT;        // state dim padded to whole lane tiles
  static constexpr int NPANEL = 2 * NT;        // 64-column panels of a B/C tile
  static constexpr int NSTAGE = NT == 1 ? 2 : 1;
  static constexpr int HB_BUFS = NT == 1 ? 2 : 1;
  static constexpr uint32_t X_BYTES = kPanel;
  static constexpr uint32_t BC_BYTES = NPANEL * kPanel;
  static constexpr uint32_t STAGE_BYTES = X_BYTES + 2 * BC_BYTES;
  static constexpr uint32_t HB_BYTES = NPAD * 128;
  static constexpr uint32_t OFF_XW = NSTAGE * STAGE_BYTES;         // [2] one per epilogue group
  static constexpr uint32_t OFF_HB = OFF_XW + 2 * kPanel;          // [HB_BUFS]
  static constexpr uint32_t OFF_SMALL = OFF_HB + HB_BUFS * HB_BYTES;
  static constexpr uint32_t OFF_V = OFF_SMALL;        // float[2][128] exp(cs_blockend - cs) delta
  static constexpr uint32_t OFF_WS = OFF_V + 1024;    // float[2][4] scan totals, then flags
  static constexpr uint32_t OFF_BAR = OFF_WS + 64;    // mbarriers
  static constexpr uint32_t OFF_TMEM = OFF_BAR + 256;
  static constexpr uint32_t SMEM = OFF_TMEM + 16;
  // TMEM columns: per epilogue group a 128-column C B^T tile, turned in place into
  // the bf16 mask operand M (columns 0..63) with Ydiag accumulated next to it
  // (columns 64..127); per group a Yoff accumulator; the state
  static constexpr uint32_t COL_Z = 0, COL_Y = 256, COL_H = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TX_BYTES = X_BYTES + 2 * BC_BYTES;
};
static_assert(Cfg<1>::SMEM <= 232448, "smem budget");
static_assert(Cfg<2>::SMEM <= 232448, "smem budget");
static_assert(Cfg<2>::COL_H + 64 * 2 <= 512, "tmem budget");

// Barriers.  Index +w is epilogue group w (tiles it with it % 2 == w).
enum Bar {
  FULL0 = 0, FULL1, EMPTY0, EMPTY1,
  CB_DONE0, CB_DONE1,       // C B^T of the group's tile is in its Z buffer (MMA -> group)
  M_READY0, M_READY1,       // mask operand written over Z (group -> MMA)
  Z_FREE0, Z_FREE1,         // the group has read Ydiag from its Z buffer (group -> MMA)
  XW_READY0, XW_READY1,     // w o x written (group -> MMA)
  PREP0, PREP1,             // state decayed in TMEM, Hb written, Ydiag read (group -> MMA)
  STATE_DONE0, STATE_DONE1, // state update of the group's tile done (MMA -> other group)
  YO_DONE0, YO_DONE1,       // Ydiag and Yoff done (MMA -> group; other group if one Hb)
  TEARDOWN, NBAR
};

struct KParams {
  Geom g;
  const void* dt;
  const float* A;
  const float* D;
  const float* den;  // optional [tokens][H]: y = num / den + D x (see tc_forward_den)
  const float* dt_bias;
  const float* init;
  const int32_t* cu;
  __nv_bfloat16* y;
  float* final_states;
  int* status;
  int units;
  int pslices;
};

struct Unit {
  int d, h, ps;
  int64_t start;
  int len, ntiles;
};

__device__ __forceinline__ Unit unit_of(const KParams& k, int u) {
  Unit U;
  U.ps = u % k.pslices;
  const int t = u / k.pslices;
  U.h = t % k.g.H;
  U.d = t / k.g.H;
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

// The stream of tiles a CTA processes: units blockIdx.x, +gridDim.x, ...; units
// without tokens contribute no tile.  Every role walks the same stream.
struct Cursor {
  int u, jt;
  bool valid;
  Unit U;
};
// The next unit with tokens after unit u in this CTA's stream (u < 0: none).
__device__ __noinline__ int next_unit_with_tiles(const KParams& kp, int u) {
  for (u += gridDim.x; u < kp.units; u += gridDim.x)
    if (unit_of(kp, u).ntiles > 0) return u;
  return -1;
}
// Advance to the next tile: within a unit only the tile index moves.
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

// Bounded wait: false (and the abort flag raised) if the phase did not complete
// within ~2 s or another role already gave up.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity,
                                           volatile int* abort_flag, int* status) {
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

// Final state row n (64 columns of the unit's P slice) from TMEM to final_states.
__device__ __noinline__ void tmem_state_to_final(const KParams& kp, uint32_t th, int d, int h,
                                                 int ps, int n) {
  float hv[kPT];
  tc_ld32(th, hv);
  tc_ld32(th + 32, hv + 32);
  tc_wait_ld();
  if (!kp.final_states || n >= kp.g.N) return;
  float* dst = kp.final_states + (((int64_t)d * kp.g.H + h) * kp.g.N + n) * kp.g.P + ps * kPT;
#pragma unroll
  for (int c = 0; c < kPT; c += 4)
    *reinterpret_cast<float4*>(dst + c) = make_float4(hv[c], hv[c + 1], hv[c + 2], hv[c + 3]);
}

// State row n on entry to a unit's first tile: the initial state (or zero) goes
// to Hb as bf16 and, decayed by the tile, into TMEM for the state update.
__device__ __noinline__ void enter_unit_row(const KParams& kp, uint32_t th, uint32_t hb_base,
                                            int d, int h, int ps, int n, float decay) {
  const float* src = (kp.init && n < kp.g.N)
                         ? kp.init + (((int64_t)d * kp.g.H + h) * kp.g.N + n) * kp.g.P + ps * kPT
                         : nullptr;
  float hv[kPT];
#pragma unroll
  for (int c = 0; c < kPT; c += 4) {
    const float4 f = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0, 0, 0, 0);
    hv[c] = f.x;
    hv[c + 1] = f.y;
    hv[c + 2] = f.z;
    hv[c + 3] = f.w;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st_shared_v4(hb_base + swz((uint32_t)n, (uint32_t)c), pack_bf16(hv[8 * c], hv[8 * c + 1]),
                 pack_bf16(hv[8 * c + 2], hv[8 * c + 3]), pack_bf16(hv[8 * c + 4], hv[8 * c + 5]),
                 pack_bf16(hv[8 * c + 6], hv[8 * c + 7]));
#pragma unroll
  for (int c = 0; c < kPT; ++c) hv[c] *= decay;
  tc_st32(th, hv);
  tc_st32(th + 32, hv + 32);
}

// Documents without tokens: their final state is their initial state (or zero).
__device__ __noinline__ void empty_units_final(const KParams& kp, int r, int nt) {
  if (!kp.final_states) return;
  for (int u = blockIdx.x; u < kp.units; u += gridDim.x) {
    const Unit U = unit_of(kp, u);
    if (U.ntiles != 0) continue;
    for (int mt = 0; mt < nt; ++mt) {
      const int n = r + 128 * mt;
      if (n >= kp.g.N) continue;
      const int64_t off = (((int64_t)U.d * kp.g.H + U.h) * kp.g.N + n) * kp.g.P + U.ps * kPT;
      for (int c = 0; c < kPT; ++c) kp.final_states[off + c] = kp.init ? kp.init[off + c] : 0.f;
    }
  }
}

// Off-diagonal column block cc (< q) of the diagonal tile for this thread's row:
// M[r, s] = Z[r, s] exp(cs_r - cs_b) v[s],  b = 32cc + 31,  v[s] = exp(cs_b - cs_s) delta_s
// (the decay factorises across the block boundary and both factors are <= 1).
// Reads C B^T from TMEM and writes M as bf16 pairs to columns 16cc..16cc+15 (in
// place: a warp handles its blocks in increasing cc, so the columns written were
// already read).
__device__ __noinline__ void mask_off(uint32_t zaddr, int cc, float cs_r, float cs_b,
                                      const float* v) {
  float zv[32];
  tc_ld32(zaddr + 32 * cc, zv);
  tc_wait_ld();
  const float u = ex2(cs_r - cs_b);
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    pk[i] = pack_bf16(zv[2 * i] * (u * v[32 * cc + 2 * i]), zv[2 * i + 1] * (u * v[32 * cc + 2 * i + 1]));
  tc_st16(zaddr + 16 * cc, pk);
}
// Diagonal 32 x 32 block of warp q: rows and columns both belong to this warp's
// lanes, so cs_s and delta_s come from the lanes by shuffle.  M[r, s] =
// Z exp(cs_r - cs_s) delta_s for s <= r, 0 above; the skip term D sits on s = r.
__device__ __noinline__ void mask_diag(uint32_t zaddr, int q, int lane, float cs, float dl,
                                       float Dh) {
  float zv[32];
  tc_ld32(zaddr + 32 * q, zv);
  tc_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float cj = __shfl_sync(0xffffffffu, cs, j);
    const float dj = __shfl_sync(0xffffffffu, dl, j);
    float m = zv[j] * ex2(cs - cj) * dj;
    if (j == lane) m += Dh;
    zv[j] = j <= lane ? m : 0.f;
  }
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(zv[2 * i], zv[2 * i + 1]);
  tc_st16(zaddr + 16 * q, pk);
}
__device__ __forceinline__ void zero_block(uint32_t zaddr, int cc) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = 0u;
  tc_st16(zaddr + 16 * cc, pk);
}


// Number of tiles this CTA processes, and the last unit of its stream with tokens.
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
// The unit with tokens that precedes unit u in this CTA's stream.
__device__ __noinline__ int prev_unit_with_tiles(const KParams& kp, int u) {
  for (u -= gridDim.x; u >= 0; u -= gridDim.x)
    if (unit_of(kp, u).ntiles > 0) return u;
  return -1;
}

// DEN: the division by a denominator folded in (kp.den set); the plain forward is DEN = false
template <int NT, bool DEN = false>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_tc_fused(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ KParams kp) {
  using C = Cfg<NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = su32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* v_all = reinterpret_cast<float*>(smem + C::OFF_V);
  float* ws_all = reinterpret_cast<float*>(smem + C::OFF_WS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_WS + 32);
  int* bad_flag = reinterpret_cast<int*>(smem + C::OFF_WS + 36);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  auto bar = [&](int i) { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
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
      const bool group = i == M_READY0 || i == M_READY1 || i == XW_READY0 || i == XW_READY1 ||
                         i == PREP0 || i == PREP1 || i == Z_FREE0 || i == Z_FREE1;
      mbar_init(bar(i), group ? 128 : 1);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(tmem_slot)),
                 "r"(C::TMEM_COLS)
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
    // ================================ TMA producer ================================
    if (lane == 0) {
      uint32_t it = 0;
      for (Cursor c = cursor_first(kp); c.valid && !*abort_flag; cursor_next(kp, c), ++it) {
        const uint32_t s = it % C::NSTAGE, k = it / C::NSTAGE;
        if (k > 0 && !wait_bar(bar(EMPTY0 + s), (k - 1) & 1, abort_flag, kp.status)) break;
        const uint32_t st = sbase + s * C::STAGE_BYTES;
        const uint32_t fb = bar(FULL0 + s);
        const int g_idx = c.U.h / (g.H / g.G);
        const int t0 = (int)(c.U.start + (int64_t)c.jt * kTile);
        SSD_CHECK(t0 >= 0 && t0 < g.tokens && g_idx < g.G && (c.U.ps + 1) * kPT <= g.P, kp.status);
        mbar_expect_tx(fb, C::TX_BYTES);
        tma_2d(st, &tm_x, fb, c.U.h * g.P + c.U.ps * kPT, t0);
#pragma unroll
        for (int q = 0; q < C::NPANEL; ++q) {
          tma_3d(st + C::X_BYTES + q * kPanel, &tm_b, fb, q * 64, g_idx, t0);
          tma_3d(st + C::X_BYTES + C::BC_BYTES + q * kPanel, &tm_c, fb, q * 64, g_idx, t0);
        }
      }
      // drain: the last fill of every stage must have landed before the CTA exits
      // (already true on the normal path; bounded to ~0.1 s on an aborted one)
      for (uint32_t s = 0; s < C::NSTAGE; ++s) {
        if (it <= s) continue;
        const uint32_t last = (it - 1 - s) / C::NSTAGE * C::NSTAGE + s;
        const uint32_t k = last / C::NSTAGE;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(FULL0 + s), k & 1) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else if (warp == 0) {
    // ================================ MMA issuer =================================
    // Event loop over three in-order streams of work: C B^T (at most two tiles ahead
    // of Ydiag, one per Z buffer), Ydiag (after the group's mask), and the state
    // update + left factors (after the group's state hand-over).  Readiness is
    // polled without blocking so that whichever group is ready is served first.
    if (lane == 0) {
      constexpr uint32_t ID_CB = idesc(128, 128, 0, 0);    // Z = C B^T, both K-major
      constexpr uint32_t ID_YOFF = idesc(128, kPT, 0, 1);  // Yoff = C Hb, Hb MN-major
      constexpr uint32_t ID_ST = idesc(128, kPT, 1, 1);    // H += B^T XW, both MN-major
      constexpr uint32_t ID_YD = idesc(128, kPT, 0, 1);    // Ydiag = M X, M in TMEM, X MN-major
      auto stage = [&](uint32_t i) { return sbase + (i % C::NSTAGE) * C::STAGE_BYTES; };
      uint32_t ncb = 0, nyd = 0, nst = 0;
      uint64_t t_last = globaltimer();
      uint32_t idle = 0;
      while (nst < ntiles) {
        bool did = false;
        // the state update is on the chain between the two epilogue groups: serve it first
        if (nst < nyd && mbar_test(bar(XW_READY0 + (nst & 1)), (nst >> 1) & 1) &&
                   mbar_test(bar(PREP0 + (nst & 1)), (nst >> 1) & 1)) {
          tc_fence_after();
          const uint32_t w = nst & 1, st = stage(nst);
          const uint32_t b_base = st + C::X_BYTES, c_base = st + C::X_BYTES + C::BC_BYTES;
          const uint32_t hb_base = sbase + C::OFF_HB + (C::HB_BUFS == 2 ? w : 0) * C::HB_BYTES;
          const uint32_t xw_base = sbase + C::OFF_XW + w * kPanel;
          auto issue_state = [&]() {
            // H += B_j^T XW : K = tokens; A = the B tile read MN-major (n), B = XW (p)
            const uint64_t dbm = sdesc(b_base, kPanel, 1024), dxw = sdesc(xw_base, kPanel, 1024);
#pragma unroll
            for (int mt = 0; mt < NT; ++mt)
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                tc_mma(tmem + C::COL_H + mt * kPT, dbm + ((2 * mt * kPanel + kk * 2048) >> 4),
                       dxw + ((kk * 2048) >> 4), ID_ST, 1);
          };
          auto issue_yoff = [&]() {
            // Yoff = C_j Hb : K = state dim; Hb rows are n (K), 128 bytes of p (MN)
            const uint64_t dc = sdesc(c_base, 16, 1024), dhb = sdesc(hb_base, C::HB_BYTES, 1024);
#pragma unroll
            for (int kk = 0; kk < C::NPAD / 16; ++kk)
              tc_mma(tmem + C::COL_Y + w * kPT, dc + (((kk >> 2) * kPanel + (kk & 3) * 32) >> 4),
                     dhb + ((kk * 2048) >> 4), ID_YOFF, kk > 0);
          };
          if (C::HB_BUFS == 2) {
            issue_state();
            tc_commit(bar(STATE_DONE0 + w));
            issue_yoff();
            tc_commit(bar(YO_DONE0 + w));
          } else {
            // one Hb buffer: the next hand-over may only overwrite it after Yoff read it
            issue_yoff();
            issue_state();
            tc_commit(bar(STATE_DONE0 + w));
            tc_commit(bar(YO_DONE0 + w));
          }
          tc_commit(bar(EMPTY0 + nst % C::NSTAGE));
          ++nst;
          did = true;
        } else if (ncb < ntiles && ncb < nyd + 2 &&
            mbar_test(bar(FULL0 + ncb % C::NSTAGE), (ncb / C::NSTAGE) & 1) &&
            (ncb < 2 || mbar_test(bar(Z_FREE0 + (ncb & 1)), ((ncb - 2) >> 1) & 1))) {
          // Z[w] = C_j B_j^T : K = state dim
          tc_fence_after();
          const uint32_t st = stage(ncb), w = ncb & 1;
          const uint64_t dc = sdesc(st + C::X_BYTES + C::BC_BYTES, 16, 1024);
          const uint64_t db = sdesc(st + C::X_BYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < C::NPAD / 16; ++kk) {
            const uint64_t off = ((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
            tc_mma(tmem + C::COL_Z + w * 128, dc + off, db + off, ID_CB, kk > 0);
          }
          tc_commit(bar(CB_DONE0 + w));
          ++ncb;
          did = true;
        } else if (nyd < ncb && mbar_test(bar(M_READY0 + (nyd & 1)), (nyd >> 1) & 1)) {
          // Ydiag = M X_j : K = tokens.  M sits in TMEM as bf16 pairs (the 16 tokens of
          // K step kk in columns 8kk..8kk+7 of the Z buffer); Ydiag goes next to it
          tc_fence_after();
          const uint32_t w = nyd & 1;
          const uint64_t dx = sdesc(stage(nyd), kPanel, 1024);
          const uint32_t z_col = tmem + C::COL_Z + w * 128;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            tc_mma_ts(z_col + 64, z_col + 8 * kk, dx + ((kk * 2048) >> 4), ID_YD, kk > 0);
          ++nyd;
          did = true;
        }
        if (did) {
          idle = 0;
          t_last = 0;
        } else if ((++idle & 15u) != 0) {
          __nanosleep(32);  // leave issue slots to the epilogue warps of this sub-partition
        } else {
          if (*abort_flag) break;
          const uint64_t now = globaltimer();
          if (t_last == 0) {
            t_last = now;
          } else if (now - t_last > 2000000000ull) {
            *abort_flag = 1;
            set_status(kp.status, SSD_ERR_TIMEOUT);
            break;
          }
        }
      }
      // every MMA this thread issued has completed once TEARDOWN fires
      tc_commit(bar(TEARDOWN));
      // bounded by time only: TMEM is freed below, so no MMA may still run then
      if (!wait_drain(bar(TEARDOWN), 0, 2000000000ull)) set_status(kp.status, SSD_ERR_TIMEOUT);
    }
  } else {
    // ==================== epilogue group w: every other tile, end to end ====================
    const int w = (warp - 2) >> 2;  // 0: tiles 0, 2, 4, ...  1: tiles 1, 3, 5, ...
    const int q = warp & 3;         // TMEM lane quarter of this warp
    const int r = q * 32 + lane;    // tile row (token) == TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t zaddr = tmem + lane_off + C::COL_Z + w * 128;
    const uint32_t yaddr = tmem + lane_off + C::COL_Y + w * kPT;
    const uint32_t xw_base = sbase + C::OFF_XW + w * kPanel;  // w o x, then the y staging tile
    const uint32_t hb_base = sbase + C::OFF_HB + (C::HB_BUFS == 2 ? w : 0) * C::HB_BYTES;
    float* vw = v_all + 128 * w;
    float* ws = ws_all + 4 * w;
    const float LOG2E = 1.4426950408889634f;
    auto sync_g = [&]() {
      if (w == 0)
        asm volatile("bar.sync 1, 128;" ::: "memory");
      else
        asm volatile("bar.sync 2, 128;" ::: "memory");
    };
    if (w == 0) empty_units_final(kp, r, NT);

    struct Pre {
      uint32_t dt;  // raw bf16 bits: converted only in E1, so the load latency stays hidden
      float A, bias, D, den;
    };
    auto prefetch = [&](const Cursor& c) -> Pre {
      Pre p{0u, 0.f, 0.f, 0.f, 1.f};
      if (!c.valid) return p;
      const int len = min(kTile, c.U.len - c.jt * kTile);
      if (r < len)
        p.dt = ld_global_u16(reinterpret_cast<const __nv_bfloat16*>(kp.dt) +
                             (c.U.start + (int64_t)c.jt * kTile + r) * g.H + c.U.h);
      p.A = kp.A[c.U.h];
      p.bias = kp.dt_bias ? kp.dt_bias[c.U.h] : 0.f;
      p.D = kp.D ? kp.D[c.U.h] : 0.f;
      if (DEN && r < len) p.den = kp.den[(c.U.start + (int64_t)c.jt * kTile + r) * g.H + c.U.h];
      return p;
    };

    bool ok = true;
    Cursor cur = cursor_first(kp);
    if (w == 1) cursor_next(kp, cur);
    Cursor nxt = cur;
    cursor_next(kp, nxt);
    cursor_next(kp, nxt);

    // E1 of a tile: delta, in-tile cumulative log decay (log2 units), the per-column
    // factor v (shared through smem), the input weight w and exp(cs) for the output.
    // With a denominator the row's skip term is D den (on the mask diagonal) and the whole
    // output row is scaled by rs = 1 / den, so y = num / den + D x; without one both
    // factors are exactly 1.
    float cs = 0.f, dl = 0.f, wr = 0.f, el = 0.f, e0 = 0.f, e1 = 0.f, e2 = 0.f, e3 = 0.f, Dh = 0.f, rs = 1.f;
    auto stage1 = [&](const Cursor& c, const Pre& p) {
      const int len = min(kTile, c.U.len - c.jt * kTile);
      float la = 0.f;
      dl = 0.f;
      if (r < len) {
        dl = softplus_f(__uint_as_float(p.dt << 16) + p.bias);
        la = dl * p.A * LOG2E;
      }
      cs = la;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, cs, o);
        if (lane >= o) cs += t;
      }
      if (lane == 31) ws[q] = cs;
      sync_g();
      e0 = ws[0];
      e1 = e0 + ws[1];
      e2 = e1 + ws[2];
      e3 = e2 + ws[3];  // block ends; e3 = cs of the tile's last row
      const float base = q == 0 ? 0.f : q == 1 ? e0 : q == 2 ? e1 : e2;
      const float cs_end = q == 0 ? e0 : q == 1 ? e1 : q == 2 ? e2 : e3;
      cs += base;
      vw[r] = ex2(cs_end - cs) * dl;
      wr = ex2(e3 - cs) * dl;  // exp(cs_last - cs) delta
      el = ex2(cs);            // exp(cs)
      Dh = DEN ? p.D * p.den : p.D;
      rs = DEN ? 1.f / p.den : 1.f;
      sync_g();
    };

    uint32_t it = w;
    if (cur.valid) stage1(cur, prefetch(cur));
    for (; cur.valid && ok; it += 2) {
      const Unit U = cur.U;
      const int jt = cur.jt;
      const int len = min(kTile, U.len - jt * kTile);
      const int64_t t0 = U.start + (int64_t)jt * kTile;
      const uint32_t k = it >> 1, s = it % C::NSTAGE;
      const Pre pn = prefetch(nxt);  // consumed by E1 of the next tile, later in this iteration

      // With two stages, stage it % 2 == w only ever holds this group's tiles, so the
      // FULL parity test is unambiguous right away.  With one stage the group sees
      // every other fill: it first waits for this tile's C B^T, which implies the
      // load landed and that the stage cannot be refilled before this tile's state
      // update, so the parity test is then unambiguous too.
      if (C::NSTAGE == 1) {
        ok = wait_bar(bar(CB_DONE0 + w), k & 1, abort_flag, kp.status);
        if (!ok) break;
      }
      ok = wait_bar(bar(FULL0 + s), (it / C::NSTAGE) & 1, abort_flag, kp.status);
      if (!ok) break;

      // ---- E4: XW = w o x_j (MN-major B operand of the state update) ----
      {
        const uint32_t xrow = sbase + s * C::STAGE_BYTES;
#pragma unroll
        for (int cidx = 0; cidx < 8; ++cidx) {
          const uint4 xv = ld_shared_v4(xrow + swz((uint32_t)r, (uint32_t)cidx));
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
          const float2 f0 = __bfloat1622float2(p2[0]), f1 = __bfloat1622float2(p2[1]);
          const float2 f2 = __bfloat1622float2(p2[2]), f3 = __bfloat1622float2(p2[3]);
          st_shared_v4(xw_base + swz((uint32_t)r, (uint32_t)cidx), pack_bf16(wr * f0.x, wr * f0.y),
                       pack_bf16(wr * f1.x, wr * f1.y), pack_bf16(wr * f2.x, wr * f2.y),
                       pack_bf16(wr * f3.x, wr * f3.y));
        }
      }
      fence_async_smem();
      mbar_arrive(bar(XW_READY0 + w));

      // ---- E2: decay mask of the diagonal block, over C B^T in TMEM ----
      if (C::NSTAGE != 1) {
        ok = wait_bar(bar(CB_DONE0 + w), k & 1, abort_flag, kp.status);
        if (!ok) break;
      }
      tc_fence_after();
      if (q > 0) mask_off(zaddr, 0, cs, e0, vw);
      if (q > 1) mask_off(zaddr, 1, cs, e1, vw);
      if (q > 2) mask_off(zaddr, 2, cs, e2, vw);
      mask_diag(zaddr, q, lane, cs, dl, Dh);
#pragma unroll 1
      for (int cc = q + 1; cc < 4; ++cc) zero_block(zaddr, cc);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(bar(M_READY0 + w));

      // ---- E3: the state entering the tile (after the previous tile's update) ----
      if (it > 0) {
        const int pb = (C::HB_BUFS == 2 ? STATE_DONE0 : YO_DONE0) + (w ^ 1);
        ok = wait_bar(bar(pb), ((it - 1) >> 1) & 1, abort_flag, kp.status);
        if (!ok) break;
      }
      tc_fence_after();
      {
        const float decay = ex2(e3);
        int pu = -1;
        if (jt == 0 && it > 0) pu = prev_unit_with_tiles(kp, cur.u);
        const Unit P = pu >= 0 ? unit_of(kp, pu) : U;
#pragma unroll 1
        for (int mt = 0; mt < NT; ++mt) {
          const int n = r + 128 * mt;
          const uint32_t th = tmem + lane_off + C::COL_H + mt * kPT;
          if (jt == 0) {
            // the previous unit's final state is still in TMEM
            if (pu >= 0) tmem_state_to_final(kp, th, P.d, P.h, P.ps, n);
            enter_unit_row(kp, th, hb_base, U.d, U.h, U.ps, n, decay);
            continue;
          }
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            float hv[32];
            tc_ld32(th + 32 * half, hv);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_shared_v4(hb_base + swz((uint32_t)n, (uint32_t)(4 * half + c)),
                           pack_bf16(hv[8 * c], hv[8 * c + 1]), pack_bf16(hv[8 * c + 2], hv[8 * c + 3]),
                           pack_bf16(hv[8 * c + 4], hv[8 * c + 5]), pack_bf16(hv[8 * c + 6], hv[8 * c + 7]));
#pragma unroll
            for (int c = 0; c < 32; ++c) hv[c] *= decay;
            tc_st32(th + 32 * half, hv);
          }
        }
      }
      tc_wait_st();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(PREP0 + w));

      // ---- E1 of this group's next tile, while the tensor cores finish this one ----
      const float el_cur = el, rs_cur = rs;
      if (nxt.valid) stage1(nxt, pn);

      // ---- E5: y = exp(cs) Yoff + Ydiag, staged in smem, coalesced stores ----
      ok = wait_bar(bar(YO_DONE0 + w), k & 1, abort_flag, kp.status);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float yo[32], yd[32];
        tc_ld32(yaddr + 32 * half, yo);
        tc_ld32(zaddr + 64 + 32 * half, yd);
        tc_wait_ld();
        float yv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) yv[j] = DEN ? fmaf(el_cur, yo[j], yd[j]) * rs_cur : fmaf(el_cur, yo[j], yd[j]);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(xw_base + swz((uint32_t)r, (uint32_t)(4 * half + c)),
                       pack_bf16(yv[8 * c + 0], yv[8 * c + 1]), pack_bf16(yv[8 * c + 2], yv[8 * c + 3]),
                       pack_bf16(yv[8 * c + 4], yv[8 * c + 5]), pack_bf16(yv[8 * c + 6], yv[8 * c + 7]));
      }
      tc_fence_before();
      mbar_arrive(bar(Z_FREE0 + w));  // Z (mask + Ydiag) and Yoff are read: next C B^T may land
      sync_g();
      {
        // 16-byte chunk e of the 128 x 128-byte tile: row e/8, chunk e%8; a warp
        // instruction covers four whole rows
        const int tid = q * 32 + lane;
        __nv_bfloat16* ybase = kp.y + (int64_t)U.h * g.P + U.ps * kPT;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = tid + 128 * i, row = e >> 3, c = e & 7;
          if (row < len && SSD_CHECK(t0 + row < g.tokens && U.h * g.P + U.ps * kPT + c * 8 + 8 <= g.H * g.P,
                                     kp.status)) {
            const uint4 v = ld_shared_v4(xw_base + swz((uint32_t)row, (uint32_t)c));
            *reinterpret_cast<uint4*>(ybase + (t0 + row) * (int64_t)g.H * g.P + c * 8) = v;
          }
        }
      }
      sync_g();  // the staging tile is read before the next tile's w o x lands there

      cur = nxt;
      cursor_next(kp, nxt);
      cursor_next(kp, nxt);
    }
    // the group that would own the next tile hands out the last unit's final state
    if (ok && ntiles > 0 && (ntiles & 1u) == (uint32_t)w && last_unit >= 0) {
      const uint32_t lt = ntiles - 1;
      const int pb = (C::HB_BUFS == 2 ? STATE_DONE0 : YO_DONE0) + (w ^ 1);
      ok = wait_bar(bar(pb), (lt >> 1) & 1, abort_flag, kp.status);
      if (ok) {
        tc_fence_after();
        const Unit L = unit_of(kp, last_unit);
#pragma unroll 1
        for (int mt = 0; mt < NT; ++mt)
          tmem_state_to_final(kp, tmem + lane_off + C::COL_H + mt * kPT, L.d, L.h, L.ps, r + 128 * mt);
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
}  // namespace

namespace tc {
namespace {
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}
}  // namespace

bool encode_bf16_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace tc

bool tc_supported(const Geom& g, const Args*) {
  if (!g.in_bf16 || !g.out_bf16) return false;
  if (g.tokens <= 0 || g.tokens > 0x7fffffffLL || g.ndocs < 1) return false;
  if (g.P % kPT != 0 || g.P > 256) return false;
  if (g.N < 16 || g.N > 256 || g.N % 16 != 0) return false;
  if (g.Q % kTile != 0) return false;
  if ((int64_t)g.ndocs * g.H * (g.P / kPT) > 0x7fffffff) return false;
  return true;
}

int tc_units(const Geom& g) { return g.ndocs * g.H * (g.P / kPT); }
int tc_kernels(const Geom&) { return 1; }
size_t tc_workspace_bytes(const Geom&) { return 256; }

namespace {

cudaError_t tc1_forward(const Geom& g, const Args& a, const float* den, int* status, cudaStream_t stream,
                        int num_sms) {
  CUtensorMap tx, tb, tc;
  const cuuint64_t T = (cuuint64_t)g.tokens;
  {
    cuuint64_t dims[2] = {(cuuint64_t)g.H * g.P, T};
    cuuint64_t str[1] = {(cuuint64_t)g.H * g.P * 2};
    cuuint32_t box[2] = {64, kTile};
    if (!tc::encode_bf16_sw128(&tx, a.x, 2, dims, str, box)) return cudaErrorInvalidValue;
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
  kp.den = den;
  kp.dt_bias = a.dt_bias;
  kp.init = a.init;
  kp.cu = a.cu;
  kp.y = reinterpret_cast<__nv_bfloat16*>(a.y);
  kp.final_states = a.final_states;
  kp.status = status;
  kp.pslices = g.P / kPT;
  kp.units = tc_units(g);
  const int grid = kp.units < num_sms ? kp.units : num_sms;
  if (den) {
    if (g.N > 128) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_fused<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<1>::SMEM);
    if (e != cudaSuccess) return e;
    ssd_tc_fused<1, true><<<grid, kThreads, Cfg<1>::SMEM, stream>>>(tx, tb, tc, kp);
  } else if (g.N <= 128) {
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_fused<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<1>::SMEM);
    if (e != cudaSuccess) return e;
    ssd_tc_fused<1><<<grid, kThreads, Cfg<1>::SMEM, stream>>>(tx, tb, tc, kp);
  } else {
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_fused<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<2>::SMEM);
    if (e != cudaSuccess) return e;
    ssd_tc_fused<2><<<grid, kThreads, Cfg<2>::SMEM, stream>>>(tx, tb, tc, kp);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_forward(const Geom& g, const Args& a, void*, int* status, cudaStream_t stream,
                       int num_sms, const TcOpts& opts) {
  if (opts.unit_columns == 128) return tc_wide_forward(g, a, status, stream, num_sms);
  // N > 128, and any shape whose wait bound or forced-timeout test is set: the kernel
  // of ssd_tc2.cu (its bounded waits take the handle's limit)
  if (tc2_supported(g) || opts.stall || opts.wait_ns != TcOpts().wait_ns)
    return tc2_forward(g, a, status, stream, num_sms, opts.wait_ns, opts.stall);
  return tc1_forward(g, a, nullptr, status, stream, num_sms);
}

bool tc_den_supported(const Geom& g, const TcOpts& opts) {
  return opts.unit_columns == 64 && !tc2_supported(g) && !opts.stall && opts.wait_ns == TcOpts().wait_ns &&
         g.N <= 128;
}

cudaError_t tc_forward_den(const Geom& g, const Args& a, const float* den, int* status, cudaStream_t stream,
                           int num_sms, const TcOpts& opts) {
  if (!den || !tc_den_supported(g, opts)) return cudaErrorInvalidValue;
  return tc1_forward(g, a, den, status, stream, num_sms);
}

}  // namespace ssd
