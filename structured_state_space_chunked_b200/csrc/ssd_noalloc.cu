// ssd_noalloc.cu -- ssd_forward_noalloc: the chunk-parallel forward pass with its
// scratch memory in a fixed, file-scope device array instead of a workspace the
// library allocates.
//
// Who needs this: callers that must not call cudaMalloc (or any allocating
// routine) on the path that runs the layer -- for example an application whose
// device memory is budgeted up front by its own allocator, or code that cannot
// afford the implicit device-wide synchronisation an allocation may cause.  Such
// a caller owns every input and output buffer; the only other device memory this
// entry point touches is `ssd_noalloc_scratch` below, which the CUDA runtime
// reserves on each device when this library's module is loaded there and keeps
// until the process exits.
//
// Host code must not use `ssd_noalloc_scratch` as a pointer: on the host that name
// is only a stand-in for the device symbol.  Its device address is looked up once
// per device with cudaGetSymbolAddress (the first call on a device does this, with
// that device current) and is then passed to the kernels.  The address is kept
// until the process exits: a device reset between calls is not supported (the
// module would be reloaded and the array could move).
//
// Every call on a device uses the same array, and it keeps whatever the previous
// call left in it.  Nothing in it has to start at zero: each call's kernels write
// every scratch element before reading it.  Two calls whose work overlaps on the
// GPU (different streams, no ordering between them) race on the array and give
// wrong results; serialise them.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ssd_internal.h"

static __device__ __align__(256) unsigned char ssd_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return SSD_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, ssd_noalloc_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SSD_OK;
}

bool is_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" SSD_API int ssd_forward_noalloc(const ssd_desc_t* desc, const void* x, const void* dt,
                                           const float* A, const void* B, const void* C,
                                           const float* D, const float* dt_bias, int chunk_size,
                                           const float* initial_states,
                                           const int32_t* cu_seqlens, int num_docs, void* y,
                                           float* final_states, int* status,
                                           ssd_stream_t stream_) {
  ssd::NvtxRange nvtx_range("ssd_forward_noalloc");
  int rc = ssd_validate_desc(desc);
  if (rc) return rc;
  const ssd_desc_t& d = *desc;
  if (chunk_size < 1 || chunk_size > 256) return SSD_ERR_INVALID_ARG;
  const bool varlen = cu_seqlens != nullptr;
  if (varlen && (d.max_docs <= 0 || d.batch != 1 || num_docs < 1 || num_docs > d.max_docs))
    return SSD_ERR_INVALID_ARG;
  const int64_t tokens = d.batch * d.seqlen;
  if (tokens > 0 && (!x || !dt || !B || !C || !y)) return SSD_ERR_INVALID_ARG;
  if (!A) return SSD_ERR_INVALID_ARG;
  const size_t ein = d.in_dtype == SSD_BF16 ? 2 : 4;
  if (!is_aligned(x, 16) || !is_aligned(B, 16) || !is_aligned(C, 16) || !is_aligned(y, 16) ||
      !is_aligned(dt, ein) || !is_aligned(A, 4) || !is_aligned(D, 4) || !is_aligned(dt_bias, 4) ||
      !is_aligned(initial_states, 16) || !is_aligned(final_states, 16) ||
      !is_aligned(cu_seqlens, 4) || !is_aligned(status, 4))
    return SSD_ERR_INVALID_ARG;

  ssd::Geom g;
  g.tokens = tokens;
  g.seqlen = d.seqlen;
  g.H = d.nheads;
  g.P = d.headdim;
  g.N = d.dstate;
  g.G = d.ngroups;
  g.Q = chunk_size;
  g.varlen = varlen ? 1 : 0;
  g.ndocs = varlen ? num_docs : (int)d.batch;
  g.nchunks_max = varlen ? (tokens + chunk_size - 1) / chunk_size + num_docs
                         : d.batch * ((d.seqlen + chunk_size - 1) / chunk_size);
  g.in_bf16 = d.in_dtype == SSD_BF16;
  g.out_bf16 = d.out_dtype == SSD_BF16;

  // problems whose scratch does not fit the fixed array are refused before any work
  if (ssd::simt_workspace_bytes(g) > (size_t)SSD_NOALLOC_SCRATCH_BYTES)
    return SSD_ERR_SCRATCH_TOO_SMALL;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSD_ERR_CUDA;
  void* scratch = nullptr;
  rc = scratch_address(dev, &scratch);
  if (rc) return rc;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (status && cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return SSD_ERR_CUDA;
  ssd::SimtWorkspace ws;
  ssd::simt_carve_workspace(g, scratch, &ws);
  ssd::Args a{x, dt, A, B, C, D, dt_bias, initial_states, cu_seqlens, y, final_states};
  const cudaError_t e = ssd::simt_forward(g, a, ws, status, stream);
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
