// ssd_tc2.cu -- fused SSD forward on the sm_100a tensor cores with the running
// state owned by a warpgroup of its own (tcgen05 + TMEM + TMA).
//
// A work unit is (document, head, 64-wide slice of the head dimension P).  A
// persistent CTA walks its units' tokens in tiles of 128.  For tile j of a unit
// ("Transformers are SSMs", paperlayer.ai summary: §6 block decomposition,
// §6.1 diagonal blocks, §6.2 low-rank blocks and the scan across chunks):
//
//   cs_l     = sum_{k<=l} delta_k A                 in-tile cumulative log decay
//   Z        = C_j B_j^T                            (128 x 128, tensor cores)
//   M[l,s]   = Z[l,s] exp(cs_l - cs_s) delta_s,  s <= l;  M[l,l] += D
//   Ydiag    = M x_j                                (tensor cores, M from TMEM)
//   dS_j     = B_j^T (w o x_j),  w_s = exp(cs_last - cs_s) delta_s
//                                                   (right factors, tensor cores)
//   S_{j+1}  = exp(cs_last) S_j + dS_j              (the scan across tiles)
//   Yoff     = C_j bf16(S_j)                        (left factors, tensor cores)
//   y        = exp(cs_l) Yoff + Ydiag
//
// The recurrence across tiles is the only serial dependence, and warpgroup S owns
// it.  N <= 128: S sits in its registers (64 columns of N rows, fp32); per tile it
// adds dS_j, which the tensor cores write into a fresh TMEM buffer, and writes the
// bf16 copy the next tile's left-factor product reads, so no product waits on the
// previous tile's update.  N = 256 (two 128-row lane tiles, too many registers): S
// stays in TMEM; per tile the warpgroup writes its bf16 copy, decays it in place, and
// the tensor cores accumulate dS_j onto it.  A chunk of Q = 128 or 256
// tokens is processed as Q/128 tiles: for Q = 256 the strictly lower 128 x 128
// block of the chunk's quadratic form goes through the same rank-N factorisation
// the decomposition uses between chunks (the mask restricted to a strictly lower
// block is rank one, §3.2.2), equal to the quadratic form up to rounding.
//
// Warps: 0-3 the state chain (S; also w o x, the B operand of dS), 4-7 and 8-11
// two epilogue groups taking alternate tiles (cumulative decay, the decay mask
// written over C B^T in TMEM as bf16, the outputs), 12 the MMA issuer and TMEM
// owner, 13 the TMA producer of B and C, 14 the TMA producer of x (a warp of its own,
// so a wait for an x slot never holds up a B/C fill).  For N = 256 B and C sit in
// separate 64 KB slots: C B^T of a tile is issued first, then dS (after which B's slot
// frees, so the next tile's B loads while this tile's left factors run), then the left
// factors (after which C's slot frees).  The issuer and producer warps run their loops
// with all 32 lanes and warp-uniform state; a predicate inside each instruction's asm
// block picks the lane that issues it, so descriptors and coordinates stay in uniform
// registers.  Every mbarrier wait is bounded; a wait that runs out records
// SSD_ERR_TIMEOUT in the status word, raises the CTA's abort flag and every role
// unwinds; before TMEM is freed the issuer waits (bounded by time only) for its
// products, and the producer for its loads.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "ssd_internal.h"
#include "tc_common.cuh"

namespace ssd {
namespace {
using namespace tc;

constexpr int kTile = 128;      // tokens per tile
constexpr int kPT = 64;         // head-dim columns per unit
constexpr int kThreads = 512;   // 16 warps
constexpr int kWarpE0 = 4, kWarpE1 = 8, kWarpMma = 12, kWarpTma = 13, kWarpX = 14;
constexpr uint32_t kBarS = 3;   // named barrier of the state warpgroup (1, 2: epilogue groups)
constexpr float kLog2e = 1.4426950408889634f;

template <int NT>
struct Cfg2 {
  static constexpr int NPAD = 128 * NT;         // state dim padded to whole lane tiles
  static constexpr int NPANEL = 2 * NT;         // 64-column panels of one B or C tile
  static constexpr int XS = 2;                  // x tile slots
  static constexpr int BS = NT == 1 ? 2 : 1;    // B/C tile slots
  static constexpr int HBS = NT == 1 ? 2 : 1;   // slots of the bf16 state copy
  static constexpr int DSB = NT == 1 ? 2 : 1;   // dS buffers in TMEM
  static constexpr uint32_t X_BYTES = kPanel;
  static constexpr uint32_t BC1_BYTES = NPANEL * kPanel;
  static constexpr uint32_t BC_BYTES = 2 * BC1_BYTES;   // B then C
  static constexpr uint32_t HB_BYTES = NPAD * 128;
  static constexpr uint32_t OFF_X = 0;
  static constexpr uint32_t OFF_BC = OFF_X + XS * X_BYTES;
  static constexpr uint32_t OFF_XW = OFF_BC + BS * BC_BYTES;      // [2]: w o x, then y staging
  static constexpr uint32_t OFF_HB = OFF_XW + 2 * kPanel;           // [HBS]
  static constexpr uint32_t OFF_V = OFF_HB + HBS * HB_BYTES;        // float[2][128]
  static constexpr uint32_t OFF_WS = OFF_V + 1024;                  // float[4][4] scan totals
  static constexpr uint32_t OFF_FLAGS = OFF_WS + 64;                // abort, bad
  static constexpr uint32_t OFF_BAR = OFF_FLAGS + 64;
  static constexpr uint32_t OFF_TMEM = OFF_BAR + 8 * 40;
  static constexpr uint32_t SMEM = OFF_TMEM + 16;
  // TMEM columns: two C B^T tiles (mask in columns 0..63, Ydiag in 64..127), two
  // left-factor accumulators, the dS buffers
  static constexpr uint32_t COL_Z = 0, COL_YO = 256, COL_DS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t SMEM_LIMIT = 232448;
};
static_assert(Cfg2<1>::SMEM <= Cfg2<1>::SMEM_LIMIT, "smem budget");
static_assert(Cfg2<2>::SMEM <= Cfg2<2>::SMEM_LIMIT, "smem budget");
static_assert(Cfg2<1>::COL_DS + Cfg2<1>::DSB * 64 <= 512, "tmem budget");
static_assert(Cfg2<2>::COL_DS + 2 * 64 <= 512, "tmem budget");

enum Bar2 {
  XFULL0 = 0, XFULL1, XEMPTY0, XEMPTY1,   // x tile slots (TMA -> readers; MMA commit -> TMA)
  BCFULL0, BCFULL1, BCEMPTY0, BCEMPTY1,   // B/C tile slots (TMA -> MMA; MMA commit -> TMA)
  CB_DONE0, CB_DONE1,     // C B^T in the group's Z buffer (MMA -> epilogue group)
  M_READY0, M_READY1,     // mask written over it (group -> MMA)
  YD_DONE0, YD_DONE1,     // Ydiag done (MMA -> group)
  XW_READY0, XW_READY1,   // w o x written (state warps -> MMA)
  DS_DONE0, DS_DONE1,     // dS of the group's tile done (MMA -> state warps and the group)
  YO_DONE0, YO_DONE1,     // left factors done (MMA -> group and state warps)
  ZFREE0, ZFREE1,         // the group read Ydiag and Yoff (group -> MMA)
  HB_READY0, HB_READY1,   // bf16 state copy written (state warps -> MMA), per slot
  DS_FREE0, DS_FREE1,     // dS buffer read (state warps -> MMA), per buffer
  XWBUF_FREE0, XWBUF_FREE1, // the group copied out y staged in its w o x buffer (group -> state warps)
  STALL,                  // nothing arrives here: the forced-timeout test waits on it
  TEARDOWN, NBAR
};
static_assert(NBAR <= 40, "barrier space");

struct KParams2 {
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
  int pslices;
  unsigned long long wait_ns;  // bound of every wait
  int stall;                   // 1: the first epilogue wait is on a barrier nothing completes
};

struct Unit {
  int d, h, ps;
  int64_t start;
  int len, ntiles;
};

__device__ __forceinline__ Unit unit_of(const KParams2& k, int u) {
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
__device__ __noinline__ int next_unit_with_tiles(const KParams2& kp, int u) {
  for (u += gridDim.x; u < kp.units; u += gridDim.x)
    if (unit_of(kp, u).ntiles > 0) return u;
  return -1;
}
__device__ __forceinline__ void cursor_next(const KParams2& kp, Cursor& c) {
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
__device__ __forceinline__ Cursor cursor_first(const KParams2& kp) {
  Cursor c;
  c.u = next_unit_with_tiles(kp, (int)blockIdx.x - (int)gridDim.x);
  c.jt = 0;
  c.valid = c.u >= 0;
  if (c.valid) c.U = unit_of(kp, c.u);
  return c;
}
__device__ __noinline__ uint32_t count_tiles(const KParams2& kp) {
  uint32_t n = 0;
  for (int u = blockIdx.x; u < kp.units; u += gridDim.x) n += (uint32_t)unit_of(kp, u).ntiles;
  return n;
}

// Bounded wait: false (and the abort flag raised) if the phase did not complete
// within kp.wait_ns or another role already gave up.
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       int* status, unsigned long long limit) {
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_try(bar, parity)) {
    if ((++n & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit) {
        *abort_flag = 1;
        set_status(status, SSD_ERR_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

// Named-barrier sync of a 128-thread group that also ANDs `ok` over the group, so
// that every thread of the group takes the same branch after it.
__device__ __forceinline__ bool group_and(uint32_t id, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 128, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(id)
      : "memory");
  return r != 0;
}

// delta and the in-tile cumulative log2 decay of row r; e0..e3 the running totals
// at the ends of the four 32-row blocks (e3: the whole tile).  One group barrier.
struct Scan {
  float cs, dl, e0, e1, e2, e3;
};
__device__ __forceinline__ bool tile_scan(uint32_t gid, float* ws, int q, int lane, bool row_valid,
                                          uint32_t dt_bits, float A, float bias, bool ok, Scan& s) {
  float la = 0.f;
  s.dl = 0.f;
  if (row_valid) {
    s.dl = softplus_f(__uint_as_float(dt_bits << 16) + bias);
    la = s.dl * A * kLog2e;
  }
  float cs = la;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_up_sync(0xffffffffu, cs, o);
    if (lane >= o) cs += t;
  }
  if (lane == 31) ws[q] = cs;
  ok = group_and(gid, ok);
  s.e0 = ws[0];
  s.e1 = s.e0 + ws[1];
  s.e2 = s.e1 + ws[2];
  s.e3 = s.e2 + ws[3];
  s.cs = cs + (q == 0 ? 0.f : q == 1 ? s.e0 : q == 2 ? s.e1 : s.e2);
  return ok;
}

struct Pre {
  uint32_t dt;  // raw bf16 bits, converted when used so the load's latency stays hidden
  float A, bias, D;
};
__device__ __forceinline__ Pre prefetch(const KParams2& kp, const Cursor& c, int r) {
  Pre p{0u, 0.f, 0.f, 0.f};
  if (!c.valid) return p;
  const int len = min(kTile, c.U.len - c.jt * kTile);
  if (r < len)
    p.dt = ld_global_u16(reinterpret_cast<const __nv_bfloat16*>(kp.dt) +
                         (c.U.start + (int64_t)c.jt * kTile + r) * kp.g.H + c.U.h);
  p.A = kp.A[c.U.h];
  p.bias = kp.dt_bias ? kp.dt_bias[c.U.h] : 0.f;
  p.D = kp.D ? kp.D[c.U.h] : 0.f;
  return p;
}

// Off-diagonal column block cc (< q) of the tile for this thread's row:
// M[r, s] = Z[r, s] exp(cs_r - cs_b) v[s],  b = 32cc + 31,  v[s] = exp(cs_b - cs_s) delta_s
// (the decay factorises across the block boundary and both factors are <= 1).
// Reads C B^T from TMEM and writes M as bf16 pairs to columns 16cc..16cc+15, in
// place: a warp handles its blocks in increasing cc, so those columns were read.
__device__ __noinline__ void mask_off(uint32_t zaddr, int cc, float cs_r, float cs_b, const float* v) {
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
// Diagonal 32 x 32 block of warp q: cs_s and delta_s come from the lanes by
// shuffle.  M[r, s] = Z exp(cs_r - cs_s) delta_s for s <= r, 0 above; D on s = r.
__device__ __noinline__ void mask_diag(uint32_t zaddr, int q, int lane, float cs, float dl, float Dh) {
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

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_tc_fused2(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ KParams2 kp) {
  using C = Cfg2<NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = su32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* v_all = reinterpret_cast<float*>(smem + C::OFF_V);
  float* ws_all = reinterpret_cast<float*>(smem + C::OFF_WS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  int* bad_flag = reinterpret_cast<int*>(smem + C::OFF_FLAGS + 4);
  // debug builds: fills of each x and B/C slot (TMA producer) and products issued
  // (MMA issuer), read by the barrier-phase checks
  volatile int* dbg = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS + 8);
  enum { DBG_XFILL = 0, DBG_BFILL = 2, DBG_NCB = 4, DBG_NDS = 5, DBG_N = 6 };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  auto bar = [&](int i) { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  const Geom& g = kp.g;
  const unsigned long long lim = kp.wait_ns;
  auto waitb = [&](int b, uint32_t parity) {
    return mbar_try(bar(b), parity) || wait_slow(bar(b), parity, abort_flag, kp.status, lim);
  };

  // ---- set-up: alignment check, cu_seqlens check, barriers, TMEM ----------------
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *bad_flag = (sbase & 1023u) != 0 ? 2 : 0;
    for (int i = 0; i < DBG_N; ++i) dbg[i] = 0;
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
                         i == ZFREE0 || i == ZFREE1 || i == HB_READY0 || i == HB_READY1 ||
                         i == DS_FREE0 || i == DS_FREE1 || i == XWBUF_FREE0 || i == XWBUF_FREE1;
      mbar_init(bar(i), group ? 128 : 1);
    }
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
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
  const uint32_t ntiles = count_tiles(kp);

  if (warp == kWarpX) {
    // ============================== TMA producer: x ==============================
    // The whole warp walks the stream (its values stay warp-uniform); one elected
    // lane issues each copy.
    uint32_t nx = 0;
    for (Cursor c = cursor_first(kp); c.valid; cursor_next(kp, c)) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int t0 = (int)(c.U.start + (int64_t)c.jt * kTile);
      {
        const uint32_t s = nx % C::XS;
        if (nx >= C::XS && !__all_sync(0xffffffffu, waitb(XEMPTY0 + s, ((nx - C::XS) / C::XS) & 1))) break;
        if (SSD_DEBUG_ON) {
          SSD_CHECK(t0 >= 0 && t0 < g.tokens && c.U.h < g.H && (c.U.ps + 1) * kPT <= g.P, kp.status);
          if (lane == 0) dbg[DBG_XFILL + s] = (int)(nx / C::XS + 1);
          __threadfence_block();
        }
        mbar_expect_tx_w(bar(XFULL0 + s), C::X_BYTES);
        tma_2d_w(sbase + C::OFF_X + s * C::X_BYTES, &tm_x, bar(XFULL0 + s), c.U.h * g.P + c.U.ps * kPT, t0);
        ++nx;
      }
    }
    for (uint32_t s = 0; s < (uint32_t)C::XS; ++s) {
      if (nx <= s) continue;
      const uint32_t last = (nx - 1 - s) / C::XS * C::XS + s;
      wait_drain(bar(XFULL0 + s), (last / C::XS) & 1, 100000000ull);
    }
  } else if (warp == kWarpTma) {
    // ============================= TMA producer: B, C =============================
    // The whole warp walks the stream (its values stay warp-uniform); one elected
    // lane issues each copy.
    uint32_t nbc = 0;
    for (Cursor c = cursor_first(kp); c.valid; cursor_next(kp, c)) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int t0 = (int)(c.U.start + (int64_t)c.jt * kTile);
      if constexpr (NT == 2) {
        // B and C in separate slots: B frees once dS and C B^T read it, C once Yoff and
        // C B^T did, so the next tile's B loads while this tile's Yoff runs
        const uint32_t st = sbase + C::OFF_BC;
        const int gi = c.U.h / (g.H / g.G);
        if (nbc >= 1 && !__all_sync(0xffffffffu, waitb(BCEMPTY0, (nbc - 1) & 1))) break;
        if (SSD_DEBUG_ON) {
          if (lane == 0) dbg[DBG_BFILL] = (int)(nbc + 1);
          __threadfence_block();
        }
        mbar_expect_tx_w(bar(BCFULL0), C::BC1_BYTES);
#pragma unroll
        for (int q = 0; q < C::NPANEL; ++q) tma_3d_w(st + q * kPanel, &tm_b, bar(BCFULL0), q * 64, gi, t0);
        if (nbc >= 1 && !__all_sync(0xffffffffu, waitb(BCEMPTY1, (nbc - 1) & 1))) break;
        if (SSD_DEBUG_ON) {
          if (lane == 0) dbg[DBG_BFILL + 1] = (int)(nbc + 1);
          __threadfence_block();
        }
        mbar_expect_tx_w(bar(BCFULL1), C::BC1_BYTES);
#pragma unroll
        for (int q = 0; q < C::NPANEL; ++q)
          tma_3d_w(st + C::BC1_BYTES + q * kPanel, &tm_c, bar(BCFULL1), q * 64, gi, t0);
        ++nbc;
      } else
      {
        const uint32_t s = nbc % C::BS;
        if (nbc >= C::BS && !__all_sync(0xffffffffu, waitb(BCEMPTY0 + s, ((nbc - C::BS) / C::BS) & 1))) break;
        const uint32_t st = sbase + C::OFF_BC + s * C::BC_BYTES;
        const int gi = c.U.h / (g.H / g.G);
        if (SSD_DEBUG_ON) {
          SSD_CHECK(gi >= 0 && gi < g.G, kp.status);
          if (lane == 0) dbg[DBG_BFILL + s] = (int)(nbc / C::BS + 1);
          __threadfence_block();
        }
        mbar_expect_tx_w(bar(BCFULL0 + s), C::BC_BYTES);
#pragma unroll
        for (int q = 0; q < C::NPANEL; ++q) {
          tma_3d_w(st + q * kPanel, &tm_b, bar(BCFULL0 + s), q * 64, gi, t0);
          tma_3d_w(st + C::BC1_BYTES + q * kPanel, &tm_c, bar(BCFULL0 + s), q * 64, gi, t0);
        }
        ++nbc;
      }
    }
    if constexpr (NT == 2) {
      if (nbc > 0) {
        wait_drain(bar(BCFULL0), (nbc - 1) & 1, 100000000ull);
        wait_drain(bar(BCFULL1), (nbc - 1) & 1, 100000000ull);
      }
    } else {
      for (uint32_t s = 0; s < (uint32_t)C::BS; ++s) {
        if (nbc <= s) continue;
        const uint32_t last = (nbc - 1 - s) / C::BS * C::BS + s;
        wait_drain(bar(BCFULL0 + s), (last / C::BS) & 1, 100000000ull);
      }
    }
  } else if (warp == kWarpMma) {
    // ================================ MMA issuer =================================
    // A non-blocking event loop over four in-order streams: dS (feeds the state
    // chain), Yoff (left factors), C B^T, Ydiag.  N <= 128: one product per pass, dS
    // first, and a B/C slot is released once the three products that read it (dS,
    // Yoff, C B^T) are issued.  N = 256: every ready product per pass in the order
    // C B^T, dS, Yoff, Ydiag, each slot's commit straight after its last reader (a
    // commit also waits for every MMA queued before it).  The whole warp runs
    // the loop with warp-uniform decisions and lane 0 issues each instruction.  Each
    // product is issued by a path specialised on the tile's parity, so every operand
    // is a loop-invariant base plus a compile-time offset.
    {
      constexpr uint32_t ID_CB = idesc(128, 128, 0, 0);    // Z = C B^T, both K-major
      constexpr uint32_t ID_YOFF = idesc(128, kPT, 0, 1);  // Yoff = C Hb, Hb MN-major
      constexpr uint32_t ID_ST = idesc(128, kPT, 1, 1);    // dS = B^T XW, both MN-major
      constexpr uint32_t ID_YD = idesc(128, kPT, 0, 1);    // Ydiag = M X, M in TMEM
      // loop-invariant descriptor bases
      const uint64_t d_bc0 = sdesc(sbase + C::OFF_BC, 16, 1024);        // K-major B (slot 0)
      const uint64_t d_bcm0 = sdesc(sbase + C::OFF_BC, kPanel, 1024);   // MN-major B (slot 0)
      const uint64_t d_x0 = sdesc(sbase + C::OFF_X, kPanel, 1024);
      const uint64_t d_xw0 = sdesc(sbase + C::OFF_XW, kPanel, 1024);
      const uint64_t d_hb0 = sdesc(sbase + C::OFF_HB, C::HB_BYTES, 1024);
      const uint32_t tm = tmem;
      auto tst = [&](int b, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_test(bar(b), parity));
      };
      // w: parity of the tile; slot offsets of the rings follow from it
      auto issue_ds = [&](auto W) {
        constexpr uint32_t w = decltype(W)::value;
        constexpr uint32_t bs = C::BS == 2 ? w : 0, ds = C::DSB == 2 ? w : 0;
        const uint64_t dbm = d_bcm0 + ((bs * C::BC_BYTES) >> 4);
        const uint64_t dxw = d_xw0 + ((w * kPanel) >> 4);
        const uint32_t dcol = tm + C::COL_DS + ds * NT * kPT;
#pragma unroll
        for (int mt = 0; mt < NT; ++mt)
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            tc_mma_w(dcol + mt * kPT, dbm + ((2 * mt * kPanel + kk * 2048) >> 4),
                     dxw + ((kk * 2048) >> 4), ID_ST, NT == 2 || kk > 0);
        tc_commit_w(bar(DS_DONE0 + w));
      };
      auto issue_yo = [&](auto W) {
        constexpr uint32_t w = decltype(W)::value;
        constexpr uint32_t bs = C::BS == 2 ? w : 0, hs = C::HBS == 2 ? w : 0;
        const uint64_t dc = d_bc0 + ((bs * C::BC_BYTES + C::BC1_BYTES) >> 4);
        const uint64_t dhb = d_hb0 + ((hs * C::HB_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::NPAD / 16; ++kk)
          tc_mma_w(tm + C::COL_YO + w * kPT, dc + (((kk >> 2) * kPanel + (kk & 3) * 32) >> 4),
                   dhb + ((kk * 2048) >> 4), ID_YOFF, kk > 0);
        tc_commit_w(bar(YO_DONE0 + w));
      };
      auto issue_cb = [&](auto W) {
        constexpr uint32_t w = decltype(W)::value;
        constexpr uint32_t bs = C::BS == 2 ? w : 0;
        const uint64_t db = d_bc0 + ((bs * C::BC_BYTES) >> 4);
        const uint64_t dc = db + (C::BC1_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < C::NPAD / 16; ++kk) {
          const uint64_t off = ((kk >> 2) * kPanel + (kk & 3) * 32) >> 4;
          tc_mma_w(tm + C::COL_Z + w * 128, dc + off, db + off, ID_CB, kk > 0);
        }
        tc_commit_w(bar(CB_DONE0 + w));
      };
      auto issue_yd = [&](auto W) {
        // Ydiag = M X_j : K = tokens.  M sits in TMEM as bf16 pairs (the 16 tokens of
        // K step kk in columns 8kk..8kk+7 of the Z buffer); Ydiag goes next to it
        constexpr uint32_t w = decltype(W)::value;
        const uint64_t dx = d_x0 + ((w * C::X_BYTES) >> 4);
        const uint32_t z_col = tm + C::COL_Z + w * 128;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          tc_mma_ts_w(z_col + 64, z_col + 8 * kk, dx + ((kk * 2048) >> 4), ID_YD, kk > 0);
        tc_commit_w(bar(YD_DONE0 + w));
      };
      using I0 = std::integral_constant<uint32_t, 0>;
      using I1 = std::integral_constant<uint32_t, 1>;
      uint32_t nds = 0, nyo = 0, ncb = 0, nyd = 0, nbc = 0, nxe = 0, ncr = 0;
      uint64_t t_last = 0;
      uint32_t idle = 0;
      while (nyd < ntiles || nds < ntiles || nyo < ntiles) {
        bool did = false;
        if constexpr (NT == 2) {
          // C B^T first (it reads B and C), then dS (B), then Yoff (C): B's slot frees
          // after dS, C's after Yoff
          auto rel_b = [&]() {  // B read by C B^T and dS
            while (nbc < nds && nbc < ncb) {
              tc_commit_w(bar(BCEMPTY0));
              ++nbc;
            }
          };
          auto rel_x = [&]() {  // x read by Ydiag and (through w o x) dS
            while (nxe < nyd && nxe < nds) {
              tc_commit_w(bar(XEMPTY0 + nxe % C::XS));
              ++nxe;
            }
          };
          auto rel_c = [&]() {  // C read by C B^T and Yoff
            while (ncr < nyo && ncr < ncb) {
              tc_commit_w(bar(BCEMPTY1));
              ++ncr;
            }
          };
          if (ncb < ntiles && tst(BCFULL0, ncb & 1) && tst(BCFULL1, ncb & 1) &&
              (ncb < 2 || tst(ZFREE0 + (ncb & 1), ((ncb - 2) >> 1) & 1))) {
            tc_fence_after();
            SSD_CHECK(dbg[DBG_BFILL] == (int)(ncb + 1) && dbg[DBG_BFILL + 1] == (int)(ncb + 1), kp.status);
            if (SSD_DEBUG_ON && lane == 0) dbg[DBG_NCB] = (int)ncb + 1;
            if (ncb & 1) issue_cb(I1{}); else issue_cb(I0{});
            ++ncb;
            did = true;
            rel_b();
            rel_c();
          }
          if (nds < ncb && tst(XW_READY0 + (nds & 1), (nds >> 1) & 1) && tst(HB_READY0, nds & 1)) {
            tc_fence_after();
            if (SSD_DEBUG_ON && lane == 0) dbg[DBG_NDS] = (int)nds + 1;
            if (nds & 1) issue_ds(I1{}); else issue_ds(I0{});
            ++nds;
            did = true;
            rel_b();  // straight after the issue: a later product's MMAs would hold the commit
            rel_x();
          }
          if (nyo < ncb && tst(HB_READY0, nyo & 1) &&
              (nyo < 2 || tst(ZFREE0 + (nyo & 1), ((nyo - 2) >> 1) & 1))) {
            tc_fence_after();
            if (nyo & 1) issue_yo(I1{}); else issue_yo(I0{});
            ++nyo;
            did = true;
            rel_c();
          }
          if (nyd < ncb && tst(M_READY0 + (nyd & 1), (nyd >> 1) & 1) &&
              tst(XFULL0 + nyd % C::XS, (nyd / C::XS) & 1)) {
            tc_fence_after();
            SSD_CHECK(dbg[DBG_XFILL + nyd % C::XS] == (int)(nyd / C::XS + 1), kp.status);
            if (nyd & 1) issue_yd(I1{}); else issue_yd(I0{});
            ++nyd;
            did = true;
            rel_x();
          }

        } else {
        // N <= 128: dS goes to a fresh buffer the state warps have read out;
        // N = 256: it accumulates onto the state the state warps decayed (HB_READY)
        if (nds < ntiles && tst(XW_READY0 + (nds & 1), (nds >> 1) & 1) &&
            tst(BCFULL0 + nds % C::BS, (nds / C::BS) & 1) &&
            (NT == 1 ? (nds < (uint32_t)C::DSB ||
                        tst(DS_FREE0 + nds % C::DSB, ((nds - C::DSB) / C::DSB) & 1))
                     : tst(HB_READY0, nds & 1))) {
          tc_fence_after();
          SSD_CHECK(dbg[DBG_BFILL + nds % C::BS] == (int)(nds / C::BS + 1), kp.status);
          // (the count is raised before the issue: the product's completion can be
          // observed before this warp would reach a store after it)
          if (SSD_DEBUG_ON && lane == 0) dbg[DBG_NDS] = (int)nds + 1;
          if (nds & 1) issue_ds(I1{}); else issue_ds(I0{});
          ++nds;
          did = true;
        } else if (nyo < ntiles && tst(HB_READY0 + nyo % C::HBS, (nyo / C::HBS) & 1) &&
                   tst(BCFULL0 + nyo % C::BS, (nyo / C::BS) & 1) &&
                   (nyo < 2 || tst(ZFREE0 + (nyo & 1), ((nyo - 2) >> 1) & 1))) {
          tc_fence_after();
          if (nyo & 1) issue_yo(I1{}); else issue_yo(I0{});
          ++nyo;
          did = true;
        } else if (ncb < ntiles && tst(BCFULL0 + ncb % C::BS, (ncb / C::BS) & 1) &&
                   (ncb < 2 || tst(ZFREE0 + (ncb & 1), ((ncb - 2) >> 1) & 1))) {
          tc_fence_after();
          // the B/C slot holds this tile's fill, not an earlier one
          SSD_CHECK(dbg[DBG_BFILL + ncb % C::BS] == (int)(ncb / C::BS + 1), kp.status);
          if (SSD_DEBUG_ON && lane == 0) dbg[DBG_NCB] = (int)ncb + 1;
          if (ncb & 1) issue_cb(I1{}); else issue_cb(I0{});
          ++ncb;
          did = true;
        } else if (nyd < ncb && tst(M_READY0 + (nyd & 1), (nyd >> 1) & 1) &&
                   tst(XFULL0 + nyd % C::XS, (nyd / C::XS) & 1)) {
          tc_fence_after();
          SSD_CHECK(dbg[DBG_XFILL + nyd % C::XS] == (int)(nyd / C::XS + 1), kp.status);
          if (nyd & 1) issue_yd(I1{}); else issue_yd(I0{});
          ++nyd;
          did = true;
        }
        while (nbc < nds && nbc < nyo && nbc < ncb) {
          tc_commit_w(bar(BCEMPTY0 + nbc % C::BS));
          ++nbc;
        }
        // an x slot is free once Ydiag read it and the state warps built w o x from it
        // (dS of the tile is issued only after that)
        while (nxe < nyd && nxe < nds) {
          tc_commit_w(bar(XEMPTY0 + nxe % C::XS));
          ++nxe;
        }
        }  // NT == 1
        if (did) {
          idle = 0;
          t_last = 0;
        } else if ((++idle & 15u) != 0) {
          __nanosleep(32);  // leave issue slots to the other warps of this sub-partition
        } else {
          if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
          const uint64_t now = globaltimer();
          if (t_last == 0) {
            t_last = now;
          } else if (__any_sync(0xffffffffu, now - t_last > lim)) {
            *abort_flag = 1;
            set_status(kp.status, SSD_ERR_TIMEOUT);
            break;
          }
        }
      }
      // every product this warp issued has completed once TEARDOWN fires; bounded by
      // time only, since TMEM is freed below
      tc_commit_w(bar(TEARDOWN));
      if (!wait_drain(bar(TEARDOWN), 0, 2000000000ull)) set_status(kp.status, SSD_ERR_TIMEOUT);
    }
  } else if (warp < kWarpE0) {
    // ======================= state warpgroup: the scan across tiles ==================
    // Thread (warp q, lane) owns state rows n = 32q + lane + 128 mt (TMEM lane quarter
    // q of every lane tile mt), 64 columns each, in registers.
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float* ws = ws_all + 8;  // two 4-float halves, alternating by tile
    // XW = w o x_j, the MN-major B operand of dS_j, w_r = exp(cs_last - cs_r) delta_r,
    // written into the w o x buffer of the tile's parity once the epilogue group has
    // copied out the y tile it staged there two tiles earlier
    auto make_xw = [&](uint32_t j, const Scan& sc, bool ok) -> bool {
      const uint32_t wb = j & 1;
      if (ok && j >= 2) ok = __all_sync(0xffffffffu, waitb(XWBUF_FREE0 + wb, ((j - 2) >> 1) & 1));
      if (ok) ok = __all_sync(0xffffffffu, waitb(XFULL0 + j % C::XS, (j / C::XS) & 1));
      if (ok) {
        const float wr = ex2(sc.e3 - sc.cs) * sc.dl;
        const uint32_t xrow = sbase + C::OFF_X + (j % C::XS) * C::X_BYTES;
        const uint32_t xw_base = sbase + C::OFF_XW + wb * kPanel;
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
        fence_async_smem();
        mbar_arrive(bar(XW_READY0 + wb));
      }
      return ok;
    };
    // documents without tokens: their final state is their initial state (or zero)
    if (kp.final_states) {
      for (int u = blockIdx.x; u < kp.units; u += gridDim.x) {
        const Unit U = unit_of(kp, u);
        if (U.ntiles != 0) continue;
        for (int mt = 0; mt < NT; ++mt) {
          const int n = r + 128 * mt;
          if (n >= g.N) continue;
          const int64_t off = (((int64_t)U.d * g.H + U.h) * g.N + n) * g.P + U.ps * kPT;
          for (int c = 0; c < kPT; c += 4)
            *reinterpret_cast<float4*>(kp.final_states + off + c) =
                kp.init ? *reinterpret_cast<const float4*>(kp.init + off + c) : make_float4(0, 0, 0, 0);
        }
      }
    }
    bool ok = true;
    Cursor cur = cursor_first(kp);
    Pre pre = prefetch(kp, cur, r);
    if constexpr (NT == 2) {
      // N = 256: the state stays in TMEM (two lane tiles of 64 columns at COL_DS) and
      // the tensor cores accumulate dS onto it; per tile these warps write the bf16
      // copy of the entering state and decay it in place for the update.
      for (uint32_t j = 0; cur.valid; ++j) {
        const Unit U = cur.U;
        const int len = min(kTile, U.len - cur.jt * kTile);
        Scan sc;
        ok = tile_scan(kBarS, ws + 4 * (j & 1), q, lane, r < len, pre.dt, pre.A, pre.bias, ok, sc);
        if (!ok) break;
        Cursor nxt = cur;
        cursor_next(kp, nxt);
        pre = prefetch(kp, nxt, r);
        // w o x of this tile first: it needs only x and the scan, and dS of the tile
        // (which frees the B/C slot) waits for it
        ok = make_xw(j, sc, ok);
        // the state after tile j-1 is complete, and its left factors read the bf16 copy
        if (ok && cur.jt > 0)
          ok = __all_sync(0xffffffffu, waitb(DS_DONE0 + ((j - 1) & 1), ((j - 1) >> 1) & 1));
        if (ok && j > 0)
          ok = __all_sync(0xffffffffu, waitb(YO_DONE0 + ((j - 1) & 1), ((j - 1) >> 1) & 1));
        if (ok) {
          tc_fence_after();
          const float decay = ex2(sc.e3);
          const uint32_t hb = sbase + C::OFF_HB;
#pragma unroll 1
          for (int mt = 0; mt < NT; ++mt) {
            const int n = r + 128 * mt;
            const uint32_t th = tmem + lane_off + C::COL_DS + mt * kPT;
            const float* src = (cur.jt == 0 && kp.init && n < g.N)
                                   ? kp.init + (((int64_t)U.d * g.H + U.h) * g.N + n) * g.P + U.ps * kPT
                                   : nullptr;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              float hv[32];
              if (cur.jt == 0) {
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                  const float4 f = src ? *reinterpret_cast<const float4*>(src + 32 * h2 + c)
                                       : make_float4(0, 0, 0, 0);
                  hv[c] = f.x;
                  hv[c + 1] = f.y;
                  hv[c + 2] = f.z;
                  hv[c + 3] = f.w;
                }
              } else {
                tc_ld32(th + 32 * h2, hv);
                tc_wait_ld();
              }
#pragma unroll
              for (int c = 0; c < 4; ++c)
                st_shared_v4(hb + swz((uint32_t)n, (uint32_t)(4 * h2 + c)),
                             pack_bf16(hv[8 * c], hv[8 * c + 1]), pack_bf16(hv[8 * c + 2], hv[8 * c + 3]),
                             pack_bf16(hv[8 * c + 4], hv[8 * c + 5]),
                             pack_bf16(hv[8 * c + 6], hv[8 * c + 7]));
#pragma unroll
              for (int c = 0; c < 32; ++c) hv[c] *= decay;
              tc_st32(th + 32 * h2, hv);
            }
          }
          tc_wait_st();
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(bar(HB_READY0));
        }
        // the unit's last tile: the final state once its update is done
        if (ok && cur.jt == U.ntiles - 1) {
          ok = __all_sync(0xffffffffu, waitb(DS_DONE0 + (j & 1), (j >> 1) & 1));
          if (ok) SSD_CHECK(dbg[DBG_NDS] >= (int)(j + 1), kp.status);
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int mt = 0; mt < NT; ++mt) {
              const int n = r + 128 * mt;
              float hv[kPT];
              tc_ld32(tmem + lane_off + C::COL_DS + mt * kPT, hv);
              tc_ld32(tmem + lane_off + C::COL_DS + mt * kPT + 32, hv + 32);
              tc_wait_ld();
              if (kp.final_states && n < g.N) {
                float* dst = kp.final_states + (((int64_t)U.d * g.H + U.h) * g.N + n) * g.P + U.ps * kPT;
#pragma unroll
                for (int c = 0; c < kPT; c += 4)
                  *reinterpret_cast<float4*>(dst + c) = make_float4(hv[c], hv[c + 1], hv[c + 2], hv[c + 3]);
              }
            }
          }
        }
        cur = nxt;
      }
    } else {
    float S[NT][kPT];
    for (uint32_t j = 0; cur.valid; ++j) {
      const Unit U = cur.U;
      const int len = min(kTile, U.len - cur.jt * kTile);
      Scan sc;
      ok = tile_scan(kBarS, ws + 4 * (j & 1), q, lane, r < len, pre.dt, pre.A, pre.bias, ok, sc);
      if (!ok) break;
      Cursor nxt = cur;
      cursor_next(kp, nxt);
      pre = prefetch(kp, nxt, r);
      if (cur.jt == 0) {
        // the state entering the unit: its initial state, or zero
#pragma unroll
        for (int mt = 0; mt < NT; ++mt) {
          const int n = r + 128 * mt;
          const float* src = (kp.init && n < g.N)
                                 ? kp.init + (((int64_t)U.d * g.H + U.h) * g.N + n) * g.P + U.ps * kPT
                                 : nullptr;
#pragma unroll
          for (int c = 0; c < kPT; c += 4) {
            const float4 f = src ? *reinterpret_cast<const float4*>(src + c) : make_float4(0, 0, 0, 0);
            S[mt][c] = f.x;
            S[mt][c + 1] = f.y;
            S[mt][c + 2] = f.z;
            S[mt][c + 3] = f.w;
          }
        }
      }
      // bf16 copy of the state entering tile j (the B operand of its left factors)
      if (j >= (uint32_t)C::HBS)
        ok = __all_sync(0xffffffffu, waitb(YO_DONE0 + ((j - C::HBS) & 1), ((j - C::HBS) >> 1) & 1));
      if (ok) {
        const uint32_t hb = sbase + C::OFF_HB + (j % C::HBS) * C::HB_BYTES;
#pragma unroll
        for (int mt = 0; mt < NT; ++mt) {
          const uint32_t n = (uint32_t)(r + 128 * mt);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(hb + swz(n, (uint32_t)c), pack_bf16(S[mt][8 * c], S[mt][8 * c + 1]),
                         pack_bf16(S[mt][8 * c + 2], S[mt][8 * c + 3]),
                         pack_bf16(S[mt][8 * c + 4], S[mt][8 * c + 5]),
                         pack_bf16(S[mt][8 * c + 6], S[mt][8 * c + 7]));
        }
        fence_async_smem();
        mbar_arrive(bar(HB_READY0 + j % C::HBS));
      }
      ok = make_xw(j, sc, ok);
      // S <- exp(cs_last) S + dS_j
      if (ok) ok = __all_sync(0xffffffffu, waitb(DS_DONE0 + (j & 1), (j >> 1) & 1));
      if (ok) SSD_CHECK(dbg[DBG_NDS] >= (int)(j + 1), kp.status);  // dS of this tile was issued
      if (ok) {
        tc_fence_after();
        const float decay = ex2(sc.e3);
        const uint32_t dcol = tmem + lane_off + C::COL_DS + (j % C::DSB) * NT * kPT;
#pragma unroll
        for (int mt = 0; mt < NT; ++mt) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            float dv[32];
            tc_ld32(dcol + mt * kPT + 32 * h2, dv);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) S[mt][32 * h2 + c] = fmaf(decay, S[mt][32 * h2 + c], dv[c]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(DS_FREE0 + j % C::DSB));
        if (cur.jt == U.ntiles - 1 && kp.final_states) {
#pragma unroll
          for (int mt = 0; mt < NT; ++mt) {
            const int n = r + 128 * mt;
            if (n >= g.N) continue;
            float* dst = kp.final_states + (((int64_t)U.d * g.H + U.h) * g.N + n) * g.P + U.ps * kPT;
#pragma unroll
            for (int c = 0; c < kPT; c += 4)
              *reinterpret_cast<float4*>(dst + c) =
                  make_float4(S[mt][c], S[mt][c + 1], S[mt][c + 2], S[mt][c + 3]);
          }
        }
      }
      cur = nxt;
    }
    }  // NT == 1
  } else if (warp < kWarpMma) {
    // ==================== epilogue group w: every other tile, end to end ====================
    const int w = warp < kWarpE1 ? 0 : 1;  // 0: tiles 0, 2, 4, ...  1: tiles 1, 3, 5, ...
    const uint32_t gid = 1 + (uint32_t)w;
    const int q = warp & 3;                // TMEM lane quarter of this warp
    const int r = q * 32 + lane;           // tile row (token) == TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t zaddr = tmem + lane_off + C::COL_Z + w * 128;
    const uint32_t yaddr = tmem + lane_off + C::COL_YO + w * kPT;
    const uint32_t xw_base = sbase + C::OFF_XW + w * kPanel;  // w o x, then the y staging tile
    float* vw = v_all + 128 * w;
    float* ws = ws_all + 4 * w;
    bool ok = true;
    Cursor cur = cursor_first(kp);
    if (w == 1) cursor_next(kp, cur);
    Pre pre = prefetch(kp, cur, r);
    if (kp.stall && w == 0 && cur.valid)
      ok = __all_sync(0xffffffffu, waitb(STALL, 0));  // runs out: the forced-timeout test
    for (uint32_t j = w; cur.valid; j += 2) {
      const Unit U = cur.U;
      const int jt = cur.jt;
      const int len = min(kTile, U.len - jt * kTile);
      const int64_t t0 = U.start + (int64_t)jt * kTile;
      const uint32_t k = j >> 1;
      // ---- E1: delta, cumulative decay, per-row and per-column factors ----
      Scan sc;
      ok = tile_scan(gid, ws, q, lane, r < len, pre.dt, pre.A, pre.bias, ok, sc);
      if (!ok) break;
      const float Dh = pre.D;
      {
        const float cs_end = q == 0 ? sc.e0 : q == 1 ? sc.e1 : q == 2 ? sc.e2 : sc.e3;
        vw[r] = ex2(cs_end - sc.cs) * sc.dl;
      }
      const float el = ex2(sc.cs);  // exp(cs)
      Cursor nxt = cur;
      cursor_next(kp, nxt);
      cursor_next(kp, nxt);
      pre = prefetch(kp, nxt, r);
      ok = group_and(gid, ok);  // vw visible to the group
      if (!ok) break;

      // ---- E2: decay mask of the diagonal block, over C B^T in TMEM ----
      ok = __all_sync(0xffffffffu, waitb(CB_DONE0 + w, k & 1));
      if (ok) {
        SSD_CHECK(dbg[DBG_NCB] >= (int)(j + 1), kp.status);
        tc_fence_after();
        if (q > 0) mask_off(zaddr, 0, sc.cs, sc.e0, vw);
        if (q > 1) mask_off(zaddr, 1, sc.cs, sc.e1, vw);
        if (q > 2) mask_off(zaddr, 2, sc.cs, sc.e2, vw);
        mask_diag(zaddr, q, lane, sc.cs, sc.dl, Dh);
#pragma unroll 1
        for (int cc = q + 1; cc < 4; ++cc) zero_block(zaddr, cc);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar(M_READY0 + w));
      }

      // ---- E5: y = exp(cs) Yoff + Ydiag, staged in smem, coalesced stores ----
      // (dS done: it read XW, whose buffer takes the y staging tile)
      if (ok)
        ok = __all_sync(0xffffffffu, waitb(YD_DONE0 + w, k & 1) && waitb(YO_DONE0 + w, k & 1) &&
                                         waitb(DS_DONE0 + w, k & 1));
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float yo[32], yd[32];
          tc_ld32(yaddr + 32 * half, yo);
          tc_ld32(zaddr + 64 + 32 * half, yd);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_shared_v4(xw_base + swz((uint32_t)r, (uint32_t)(4 * half + c)),
                         pack_bf16(fmaf(el, yo[8 * c + 0], yd[8 * c + 0]), fmaf(el, yo[8 * c + 1], yd[8 * c + 1])),
                         pack_bf16(fmaf(el, yo[8 * c + 2], yd[8 * c + 2]), fmaf(el, yo[8 * c + 3], yd[8 * c + 3])),
                         pack_bf16(fmaf(el, yo[8 * c + 4], yd[8 * c + 4]), fmaf(el, yo[8 * c + 5], yd[8 * c + 5])),
                         pack_bf16(fmaf(el, yo[8 * c + 6], yd[8 * c + 6]), fmaf(el, yo[8 * c + 7], yd[8 * c + 7])));
        }
        tc_fence_before();
        mbar_arrive(bar(ZFREE0 + w));  // Z (mask + Ydiag) and Yoff read: the next products may land
      }
      ok = group_and(gid, ok);
      if (!ok) break;
      {
        // 16-byte chunk e of the 128 x 128-byte tile: row e/8, chunk e%8; a warp
        // instruction covers four whole rows.
        __nv_bfloat16* ybase = kp.y + (int64_t)U.h * g.P + U.ps * kPT;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = r + 128 * i, row = e >> 3, c = e & 7;
          if (row < len && SSD_CHECK(t0 + row < g.tokens && U.h * g.P + U.ps * kPT + c * 8 + 8 <= g.H * g.P,
                                     kp.status)) {
            const uint4 v = ld_shared_v4(xw_base + swz((uint32_t)row, (uint32_t)c));
            *reinterpret_cast<uint4*>(ybase + (t0 + row) * (int64_t)g.H * g.P + c * 8) = v;
          }
        }
        mbar_arrive(bar(XWBUF_FREE0 + w));  // the buffer takes w o x of tile j + 2
      }
      cur = nxt;
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace

// Shapes this kernel takes: the 64-column tensor-core path with N > 128 (two lane
// tiles of state).  For N <= 128 the kernel of ssd_tc.cu measured faster on every
// benchmark shape, so it keeps those (this kernel computes them as well).
bool tc2_supported(const Geom& g) { return g.N > 128 && g.N <= 256; }

cudaError_t tc2_forward(const Geom& g, const Args& a, int* status, cudaStream_t stream, int num_sms,
                        unsigned long long wait_ns, int stall) {
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
  KParams2 kp;
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
  kp.pslices = g.P / kPT;
  kp.units = g.ndocs * g.H * kp.pslices;
  kp.wait_ns = wait_ns;
  kp.stall = stall;
  const int grid = kp.units < num_sms ? kp.units : num_sms;
  if (g.N <= 128) {
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_fused2<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg2<1>::SMEM);
    if (e != cudaSuccess) return e;
    ssd_tc_fused2<1><<<grid, kThreads, Cfg2<1>::SMEM, stream>>>(tx, tb, tc, kp);
  } else {
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_fused2<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg2<2>::SMEM);
    if (e != cudaSuccess) return e;
    ssd_tc_fused2<2><<<grid, kThreads, Cfg2<2>::SMEM, stream>>>(tx, tb, tc, kp);
  }
  return cudaGetLastError();
}

}  // namespace ssd
