// ssd_internal.h -- shared declarations of the CUDA library (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

#include <nvtx3/nvToolsExt.h>

namespace ssd {

// Problem geometry of one ssd_forward call, passed by value to kernels.
struct Geom {
  int64_t tokens;      // batch * seqlen
  int64_t seqlen;      // rows of batch mode
  int H, P, N, G;      // heads, head dim, state dim, groups
  int Q;               // chunk length
  int ndocs;           // documents (batch rows or cu_seqlens entries)
  int varlen;          // 1: documents come from cu_seqlens
  int64_t nchunks_max; // chunk slots (upper bound for varlen)
  int in_bf16, out_bf16;
};

// Pointers of one ssd_forward call.
struct Args {
  const void* x;
  const void* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  const float* dt_bias;
  const float* init;
  const int32_t* cu;
  void* y;
  float* final_states;
};

// An NVTX range around the launches of one entry point (visible in Nsight timelines;
// without a profiling tool attached a push/pop costs a few nanoseconds).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Device status word values are the negative SSD_ERR_* codes; 0 = ok.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Debug builds (-DSSD_DEBUG, `build.py --debug`): device-side checks of indices and
// barrier phases.  A failed check records SSD_ERR_DEBUG_CHECK in the status word and
// the source line in the word after it, and the access it guards is skipped where the
// call site says so; it never traps.  Release builds compile the checks away.
#ifdef SSD_DEBUG
#define SSD_DEBUG_ON 1
__device__ __forceinline__ bool debug_check(bool ok, int* status, int line) {
  if (!ok && status) {
    if (atomicCAS(status, 0, SSD_ERR_DEBUG_CHECK) == 0) status[1] = line;
  }
  return ok;
}
#define SSD_CHECK(cond, status) ::ssd::debug_check((cond), (status), __LINE__)
#else
#define SSD_DEBUG_ON 0
#define SSD_CHECK(cond, status) true
#endif

__device__ __forceinline__ float load_f(const void* p, int64_t i, int bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
              : reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_f(void* p, int64_t i, float v, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p)[i] = v;
}

// softplus in fp32; for z > 20 the correction log1p(exp(-z)) < 2.1e-9 is dropped.
__device__ __forceinline__ float softplus_f(float z) {
  return z > 20.f ? z : log1pf(expf(z));
}

// ---- SIMT (chunk-parallel) path -------------------------------------------------
struct SimtWorkspace {
  float* cs;          // [H, nchunks, Q] inclusive cumsum of delta*A within the chunk
  float* delta;       // [H, nchunks, Q] delta (0 for padding positions)
  float* states;      // [nchunks, H, N, P] chunk state, then state entering the chunk
  int* chunk_doc;     // [nchunks] varlen: document of chunk k
  int* doc_first;     // [ndocs + 1] varlen: first chunk of each document
  int* total_chunks;  // [1] varlen: number of chunks in use
};

size_t simt_workspace_bytes(const Geom& g);
void simt_carve_workspace(const Geom& g, void* base, SimtWorkspace* ws);
int simt_kernels(const Geom& g);
cudaError_t simt_forward(const Geom& g, const Args& a, const SimtWorkspace& ws, int* status,
                         cudaStream_t stream);

// ---- tensor-core (tcgen05) path -------------------------------------------------
// Launch options of the tensor-core forward (handle options of ssd_set_option).
struct TcOpts {
  int unit_columns = 64;                      // 64 or 128 (ssd_tc_wide.cu)
  unsigned long long wait_ns = 2000000000ull; // bound of every device-side wait
  int stall = 0;                              // 1: forced-timeout test (ssd_tc2.cu)
};
bool tc_supported(const Geom& g, const Args* a);
int tc_units(const Geom& g);
int tc_kernels(const Geom& g);
size_t tc_workspace_bytes(const Geom& g);
cudaError_t tc_forward(const Geom& g, const Args& a, void* workspace, int* status,
                       cudaStream_t stream, int num_sms, const TcOpts& opts);
// the kernel with the state chain in registers (ssd_tc2.cu): N <= 128
bool tc2_supported(const Geom& g);
cudaError_t tc2_forward(const Geom& g, const Args& a, int* status, cudaStream_t stream, int num_sms,
                        unsigned long long wait_ns, int stall);
// 128-column units (ssd_tc_wide.cu): tc_forward with unit_columns == 128
bool tc_wide_supported(const Geom& g);
int tc_wide_units(const Geom& g);
cudaError_t tc_wide_forward(const Geom& g, const Args& a, int* status, cudaStream_t stream,
                            int num_sms);

}  // namespace ssd
