// ssd_api.cu -- the C ABI declared in include/ssd.h: argument checks, path
// selection, workspace management and launches.  All compute runs in the
// kernels of ssd_simt.cu, ssd_tc.cu, ssd_tc_wide.cu, ssd_bwd.cu and ssd_ext.cu.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "ssd_bwd.h"
#include "ssd_ext.h"
#include "ssd_internal.h"

struct ssd_handle_s {
  ssd_desc_t desc;
  int device;
  int num_sms;
  int force_path;
  int tc_unit_columns;  // 64 or 128
  unsigned long long wait_ns;  // bound of every device-side wait of the tensor-core kernel
  int force_timeout;    // 1: the tensor-core kernel's first epilogue wait runs out (test)
  int* status;          // device status word (first error code, 0 = ok)
  void* ws;             // stream-ordered workspace
  size_t ws_bytes;
  void* io;             // device buffers of ssd_forward_host
  size_t io_bytes;
  // ssd_forward_ext's second stream: the denominator runs there beside the numerator
  // (forked after the feature maps, joined before the normalisation); made on first use
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
};

namespace {

using ssd::Geom;

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t elem_bytes(int dt) { return dt == SSD_BF16 ? 2 : 4; }

int make_geom(const ssd_desc_t& d, int chunk_size, bool varlen, int num_docs, Geom* g) {
  g->tokens = d.batch * d.seqlen;
  g->seqlen = d.seqlen;
  g->H = d.nheads;
  g->P = d.headdim;
  g->N = d.dstate;
  g->G = d.ngroups;
  g->Q = chunk_size;
  g->varlen = varlen ? 1 : 0;
  g->ndocs = varlen ? num_docs : (int)d.batch;
  if (varlen)
    g->nchunks_max = (g->tokens + chunk_size - 1) / chunk_size + num_docs;
  else
    g->nchunks_max = d.batch * ((d.seqlen + chunk_size - 1) / chunk_size);
  g->in_bf16 = d.in_dtype == SSD_BF16;
  g->out_bf16 = d.out_dtype == SSD_BF16;
  return SSD_OK;
}

int check_call(const ssd_desc_t& d, int chunk_size, const int32_t* cu, int num_docs) {
  if (chunk_size < 1 || chunk_size > 256) return SSD_ERR_INVALID_ARG;
  if (cu) {
    if (d.max_docs <= 0 || d.batch != 1) return SSD_ERR_INVALID_ARG;
    if (num_docs < 1 || num_docs > d.max_docs) return SSD_ERR_INVALID_ARG;
  }
  return SSD_OK;
}

int choose_path(const ssd_desc_t& d, const Geom& g, int force) {
  const bool tc = ssd::tc_supported(g, nullptr);
  if (force == SSD_PATH_SIMT) return SSD_PATH_SIMT;
  if (force == SSD_PATH_TC) return tc ? SSD_PATH_TC : SSD_ERR_UNSUPPORTED;
  (void)d;
  return tc ? SSD_PATH_TC : SSD_PATH_SIMT;
}

size_t workspace_for(const Geom& g, int path) {
  return path == SSD_PATH_TC ? ssd::tc_workspace_bytes(g) : ssd::simt_workspace_bytes(g);
}

int cuda_rc(cudaError_t e) {
  if (e == cudaSuccess) return SSD_OK;
  if (e == cudaErrorMemoryAllocation) return SSD_ERR_OOM;
  return SSD_ERR_CUDA;
}

ssd::TcOpts tc_opts(const ssd_handle_s* h) {
  ssd::TcOpts o;
  o.unit_columns = h->tc_unit_columns;
  o.wait_ns = h->wait_ns;
  o.stall = h->force_timeout;
  return o;
}

}  // namespace

extern "C" {

int ssd_validate_desc(const ssd_desc_t* d) {
  if (!d) return SSD_ERR_INVALID_ARG;
  if (d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->headdim <= 0 || d->dstate <= 0 ||
      d->ngroups <= 0)
    return SSD_ERR_INVALID_ARG;
  if (d->in_dtype != SSD_F32 && d->in_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (d->out_dtype != SSD_F32 && d->out_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (d->flags != 0 || d->max_docs < 0) return SSD_ERR_INVALID_ARG;
  if (d->max_docs > 0 && d->batch != 1) return SSD_ERR_INVALID_ARG;
  if (d->batch * d->seqlen > ((int64_t)1 << 40)) return SSD_ERR_UNSUPPORTED;
  if (d->nheads % d->ngroups != 0) return SSD_ERR_UNSUPPORTED;
  if (d->headdim > 256 || d->dstate > 256) return SSD_ERR_UNSUPPORTED;
  return SSD_OK;
}

int ssd_plan(const ssd_desc_t* desc, int chunk_size, int num_docs, ssd_plan_t* out) {
  int rc = ssd_validate_desc(desc);
  if (rc) return rc;
  if (!out) return SSD_ERR_INVALID_ARG;
  const bool varlen = num_docs > 0;
  rc = check_call(*desc, chunk_size, varlen ? (const int32_t*)1 : nullptr, num_docs);
  if (rc) return rc;
  Geom g;
  make_geom(*desc, chunk_size, varlen, num_docs, &g);
  const int path = choose_path(*desc, g, SSD_PATH_AUTO);
  memset(out, 0, sizeof(*out));
  out->path = path;
  out->num_docs = g.ndocs;
  out->num_chunks_max = g.nchunks_max;
  out->workspace_bytes = (int64_t)workspace_for(g, path);
  out->units = path == SSD_PATH_TC ? ssd::tc_units(g) : 0;
  out->kernels = path == SSD_PATH_TC ? ssd::tc_kernels(g) : ssd::simt_kernels(g);
  return SSD_OK;
}

int ssd_create(const ssd_desc_t* desc, ssd_handle_t* out) {
  int rc = ssd_validate_desc(desc);
  if (rc) return rc;
  if (!out) return SSD_ERR_INVALID_ARG;
  *out = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSD_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SSD_ERR_CUDA;
  ssd_handle_s* h = new (std::nothrow) ssd_handle_s();
  if (!h) return SSD_ERR_OOM;
  h->desc = *desc;
  h->device = dev;
  h->num_sms = sms;
  h->force_path = SSD_PATH_AUTO;
  h->tc_unit_columns = 64;
  h->wait_ns = 2000000000ull;
  h->force_timeout = 0;
  cudaError_t e = cudaMalloc(&h->status, sizeof(int) * 4);
  if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(int) * 4);
  if (e != cudaSuccess) {
    if (h->status) cudaFree(h->status);
    delete h;
    return cuda_rc(e);
  }
  *out = h;
  return SSD_OK;
}

int ssd_set_option(ssd_handle_t h, int option, int value) {
  if (!h) return SSD_ERR_INVALID_ARG;
  if (option == SSD_OPT_FORCE_PATH) {
    if (value != SSD_PATH_AUTO && value != SSD_PATH_SIMT && value != SSD_PATH_TC)
      return SSD_ERR_INVALID_ARG;
    h->force_path = value;
    return SSD_OK;
  }
  if (option == SSD_OPT_TC_UNIT_COLUMNS) {
    if (value != 64 && value != 128) return SSD_ERR_INVALID_ARG;
    h->tc_unit_columns = value;
    return SSD_OK;
  }
  if (option == SSD_OPT_WAIT_LIMIT_US) {
    if (value < 1 || value > 60000000) return SSD_ERR_INVALID_ARG;
    h->wait_ns = 1000ull * (unsigned long long)value;
    return SSD_OK;
  }
  if (option == SSD_OPT_TEST_FORCE_TIMEOUT) {
    if (value != 0 && value != 1) return SSD_ERR_INVALID_ARG;
    h->force_timeout = value;
    return SSD_OK;
  }
  return SSD_ERR_INVALID_ARG;
}

int ssd_forward(ssd_handle_t h, const void* x, const void* dt, const float* A, const void* B,
                const void* C, const float* D, const float* dt_bias, int chunk_size,
                const float* initial_states, const int32_t* cu_seqlens, int num_docs, void* y,
                float* final_states, ssd_stream_t stream_) {
  ssd::NvtxRange nvtx_range("ssd_forward");
  if (!h) return SSD_ERR_INVALID_ARG;
  const ssd_desc_t& d = h->desc;
  int rc = check_call(d, chunk_size, cu_seqlens, num_docs);
  if (rc) return rc;
  const int64_t tokens = d.batch * d.seqlen;
  if (tokens > 0 && (!x || !dt || !B || !C || !y)) return SSD_ERR_INVALID_ARG;
  if (!A) return SSD_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) ||
      !aligned(dt, elem_bytes(d.in_dtype)) || !aligned(A, 4) || !aligned(D, 4) ||
      !aligned(dt_bias, 4) || !aligned(initial_states, 16) || !aligned(final_states, 16) ||
      !aligned(cu_seqlens, 4))
    return SSD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  Geom g;
  make_geom(d, chunk_size, cu_seqlens != nullptr, num_docs, &g);
  const int path = choose_path(d, g, h->force_path);
  if (path < 0) return path;
  if (path == SSD_PATH_TC && h->tc_unit_columns == 128 && !ssd::tc_wide_supported(g))
    return SSD_ERR_UNSUPPORTED;

  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return SSD_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return SSD_ERR_CUDA;

  const size_t need = workspace_for(g, path);
  if (need > h->ws_bytes) {
    if (h->ws) cudaFreeAsync(h->ws, stream);
    h->ws = nullptr;
    h->ws_bytes = 0;
    cudaError_t e = cudaMallocAsync(&h->ws, need, stream);
    if (e != cudaSuccess) {
      h->ws = nullptr;
      if (cur != h->device) cudaSetDevice(cur);
      return cuda_rc(e);
    }
    h->ws_bytes = need;
  }
  ssd::Args a{x, dt, A, B, C, D, dt_bias, initial_states, cu_seqlens, y, final_states};
  cudaError_t e;
  if (path == SSD_PATH_TC) {
    e = ssd::tc_forward(g, a, h->ws, h->status, stream, h->num_sms, tc_opts(h));
  } else {
    ssd::SimtWorkspace ws;
    ssd::simt_carve_workspace(g, h->ws, &ws);
    e = ssd::simt_forward(g, a, ws, h->status, stream);
  }
  if (cur != h->device) cudaSetDevice(cur);
  return cuda_rc(e);
}

int ssd_backward(ssd_handle_t h, const void* x, const void* dt, const float* A, const void* B,
                 const void* C, const float* D, const float* dt_bias, const float* initial_states,
                 const int32_t* cu_seqlens, int num_docs, const void* dy, const float* dfinal_states,
                 float* dx, float* ddt, float* dA, float* dB, float* dC, float* dD, float* ddt_bias,
                 float* dinitial_states, ssd_stream_t stream_) {
  ssd::NvtxRange nvtx_range("ssd_backward");
  if (!h) return SSD_ERR_INVALID_ARG;
  const ssd_desc_t& d = h->desc;
  int rc = check_call(d, ssd::kBwdQ, cu_seqlens, num_docs);
  if (rc) return rc;
  const int64_t tokens = d.batch * d.seqlen;
  if (tokens > 0 && (!x || !dt || !B || !C || !dy || !dx || !ddt || !dB || !dC))
    return SSD_ERR_INVALID_ARG;
  if (!A || !dA) return SSD_ERR_INVALID_ARG;
  const size_t ei = elem_bytes(d.in_dtype), eo = elem_bytes(d.out_dtype);
  if (!aligned(x, ei) || !aligned(dt, ei) || !aligned(B, ei) || !aligned(C, ei) || !aligned(dy, eo) ||
      !aligned(A, 4) || !aligned(D, 4) || !aligned(dt_bias, 4) || !aligned(initial_states, 4) ||
      !aligned(dfinal_states, 4) || !aligned(dx, 4) || !aligned(ddt, 4) || !aligned(dA, 4) ||
      !aligned(dB, 4) || !aligned(dC, 4) || !aligned(dD, 4) || !aligned(ddt_bias, 4) ||
      !aligned(dinitial_states, 4) || !aligned(cu_seqlens, 4))
    return SSD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  ssd::Args a{x, dt, A, B, C, D, dt_bias, initial_states, cu_seqlens, nullptr, nullptr};
  ssd::GradArgs ga{dy, dfinal_states, dx, ddt, dA, dB, dC, dD, ddt_bias, dinitial_states};
  Geom g;
  make_geom(d, ssd::kBwdTcQ, cu_seqlens != nullptr, num_docs, &g);
  if (!ssd::bwd_tc_eligible(g, a, ga)) make_geom(d, ssd::kBwdQ, cu_seqlens != nullptr, num_docs, &g);

  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return SSD_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return SSD_ERR_CUDA;
  const size_t need = ssd::bwd_workspace_bytes(g);
  if (need > h->ws_bytes) {
    if (h->ws) cudaFreeAsync(h->ws, stream);
    h->ws = nullptr;
    h->ws_bytes = 0;
    cudaError_t e = cudaMallocAsync(&h->ws, need, stream);
    if (e != cudaSuccess) {
      h->ws = nullptr;
      if (cur != h->device) cudaSetDevice(cur);
      return cuda_rc(e);
    }
    h->ws_bytes = need;
  }
  cudaError_t e = ssd::bwd_run(g, a, ga, h->ws, h->status, stream);
  if (cur != h->device) cudaSetDevice(cur);
  return cuda_rc(e);
}

int ssd_feature_map_dim(int kind, int dstate) {
  if (dstate < 1) return -1;
  return ssd::fmap_dim(kind, dstate);
}

int ssd_forward_ext(ssd_handle_t h, const void* x, const void* dt, const float* A, const void* B,
                    const void* C, const float* D, const float* dt_bias, int chunk_size,
                    const int32_t* cu_seqlens, int num_docs, int feature_map, int normalize, void* y,
                    float* final_states, ssd_stream_t stream_) {
  ssd::NvtxRange nvtx_range("ssd_forward_ext");
  if (!h) return SSD_ERR_INVALID_ARG;
  const ssd_desc_t& d = h->desc;
  int rc = check_call(d, chunk_size, cu_seqlens, num_docs);
  if (rc) return rc;
  const int N2 = ssd::fmap_dim(feature_map, (int)d.dstate);
  if (N2 < 1 || N2 > 65536 || (normalize != 0 && normalize != 1)) return SSD_ERR_INVALID_ARG;
  const int64_t tokens = d.batch * d.seqlen;
  if (tokens > 0 && (!x || !dt || !B || !C || !y)) return SSD_ERR_INVALID_ARG;
  if (!A) return SSD_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(B, elem_bytes(d.in_dtype)) || !aligned(C, elem_bytes(d.in_dtype)) ||
      !aligned(y, 16) || !aligned(dt, elem_bytes(d.in_dtype)) || !aligned(A, 4) || !aligned(D, 4) ||
      !aligned(dt_bias, 4) || !aligned(final_states, 16) || !aligned(cu_seqlens, 4))
    return SSD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  ssd_desc_t d2 = d;
  d2.dstate = N2;
  Geom g;
  make_geom(d2, chunk_size, cu_seqlens != nullptr, num_docs, &g);
  const int path = choose_path(d2, g, h->force_path);
  if (path < 0) return path;
  if (path == SSD_PATH_TC && h->tc_unit_columns == 128 && !ssd::tc_wide_supported(g))
    return SSD_ERR_UNSUPPORTED;
  if (normalize && !ssd::den_scan_supported(N2)) return SSD_ERR_UNSUPPORTED;
  // the denominator's geometry: one column, chunks of kDenQ tokens
  ssd_desc_t dd = d2;
  dd.headdim = 1;
  Geom gd;
  make_geom(dd, ssd::kDenQ, cu_seqlens != nullptr, num_docs, &gd);

  const size_t es = elem_bytes(d.in_dtype);
  auto al = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const size_t b_bc = al(es * (size_t)tokens * d.ngroups * N2);
  const size_t b_den = normalize ? al(sizeof(float) * (size_t)tokens * d.nheads) : 0;
  const size_t b_fwd = al(workspace_for(g, path));
  const size_t b_dws = normalize ? al(ssd::simt_workspace_bytes(gd)) : 0;
  const size_t need = 2 * b_bc + b_den + b_fwd + b_dws;

  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return SSD_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return SSD_ERR_CUDA;
  if (need > h->ws_bytes) {
    if (h->ws) cudaFreeAsync(h->ws, stream);
    h->ws = nullptr;
    h->ws_bytes = 0;
    cudaError_t e = cudaMallocAsync(&h->ws, need, stream);
    if (e != cudaSuccess) {
      h->ws = nullptr;
      if (cur != h->device) cudaSetDevice(cur);
      return cuda_rc(e);
    }
    h->ws_bytes = need;
  }
  char* base = static_cast<char*>(h->ws);
  void* B2 = base;
  void* C2 = base + b_bc;
  float* den = reinterpret_cast<float*>(base + 2 * b_bc);
  void* fws = base + 2 * b_bc + b_den;
  void* dws = base + 2 * b_bc + b_den + b_fwd;
  const int bf = d.in_dtype == SSD_BF16;
  const int64_t rows = tokens * d.ngroups;
  cudaError_t e = ssd::fmap_apply(feature_map, rows, (int)d.dstate, N2, bf, B, B2, C, C2, stream);
  // Two ways to normalise.  When the numerator kernel leaves at least a quarter of the SMs
  // idle (fewer units than 3/4 of the SMs), the denominator runs beside it on the second
  // stream and a last pass divides y.  Otherwise the denominator runs first and the
  // numerator kernel divides in its output epilogue, which saves the pass over y.
  if (normalize && path == SSD_PATH_TC && ssd::tc_den_supported(g, tc_opts(h)) &&
      4 * (int64_t)ssd::tc_units(g) > 3 * (int64_t)h->num_sms) {
    if (e == cudaSuccess) e = ssd::den_scan(gd, cu_seqlens, dws, h->status, dt, A, dt_bias, B2, C2, den, stream);
    ssd::Args a{x, dt, A, B2, C2, D, dt_bias, nullptr, cu_seqlens, y, final_states};
    if (e == cudaSuccess) e = ssd::tc_forward_den(g, a, den, h->status, stream, h->num_sms, tc_opts(h));
    if (cur != h->device) cudaSetDevice(cur);
    return cuda_rc(e);
  }
  if (normalize && e == cudaSuccess && !h->side) {
    // all three or none, so a failed creation leaves the handle as it was
    cudaStream_t sd = nullptr;
    cudaEvent_t ef = nullptr, ejn = nullptr;
    e = cudaStreamCreateWithFlags(&sd, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ef, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ejn, cudaEventDisableTiming);
    if (e == cudaSuccess) {
      h->side = sd;
      h->ev_fork = ef;
      h->ev_join = ejn;
    } else {
      if (ejn) cudaEventDestroy(ejn);
      if (ef) cudaEventDestroy(ef);
      if (sd) cudaStreamDestroy(sd);
    }
  }
  if (normalize && e == cudaSuccess) e = cudaEventRecord(h->ev_fork, stream);
  // the numerator (D added after the division when normalising)
  ssd::Args a{x, dt, A, B2, C2, normalize ? nullptr : D, dt_bias, nullptr, cu_seqlens, y, final_states};
  if (e == cudaSuccess) {
    if (path == SSD_PATH_TC) {
      e = ssd::tc_forward(g, a, fws, h->status, stream, h->num_sms, tc_opts(h));
    } else {
      ssd::SimtWorkspace ws;
      ssd::simt_carve_workspace(g, fws, &ws);
      e = ssd::simt_forward(g, a, ws, h->status, stream);
    }
  }
  if (normalize && e == cudaSuccess) {
    // the denominator on the side stream, its chain beside the numerator's kernel
    e = cudaStreamWaitEvent(h->side, h->ev_fork, 0);
    if (e == cudaSuccess) e = ssd::den_scan(gd, cu_seqlens, dws, h->status, dt, A, dt_bias, B2, C2, den, h->side);
    // the join is recorded even after a failed launch, so the caller's stream never waits on
    // an event of an earlier call
    const cudaError_t ej = cudaEventRecord(h->ev_join, h->side);
    if (e == cudaSuccess) e = ej;
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, h->ev_join, 0);
    if (e == cudaSuccess)
      e = ssd::normalize_apply(tokens, (int)d.nheads, (int)d.headdim, d.out_dtype == SSD_BF16, bf, y,
                               den, x, D, stream);
  }
  if (cur != h->device) cudaSetDevice(cur);
  return cuda_rc(e);
}

int ssd_forward_host(ssd_handle_t h, const void* x, const void* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* dt_bias,
                     int chunk_size, const float* initial_states, const int32_t* cu_seqlens,
                     int num_docs, void* y, float* final_states, ssd_stream_t stream_) {
  ssd::NvtxRange nvtx_range("ssd_forward_host");
  if (!h) return SSD_ERR_INVALID_ARG;
  const ssd_desc_t& d = h->desc;
  int rc = check_call(d, chunk_size, cu_seqlens, num_docs);
  if (rc) return rc;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int64_t T = d.batch * d.seqlen;
  const int ndocs = cu_seqlens ? num_docs : (int)d.batch;
  const int maxdocs = d.max_docs > 0 ? d.max_docs : (int)d.batch;
  const size_t ein = elem_bytes(d.in_dtype), eout = elem_bytes(d.out_dtype);
  const size_t bx = (size_t)T * d.nheads * d.headdim * ein;
  const size_t bdt = (size_t)T * d.nheads * ein;
  const size_t bbc = (size_t)T * d.ngroups * d.dstate * ein;
  const size_t bh = sizeof(float) * d.nheads;
  const size_t by = (size_t)T * d.nheads * d.headdim * eout;
  const size_t bst = sizeof(float) * (size_t)maxdocs * d.nheads * d.dstate * d.headdim;
  const size_t bcu = sizeof(int32_t) * ((size_t)maxdocs + 1);
  auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const size_t off_x = 0, off_dt = off_x + up(bx), off_B = off_dt + up(bdt),
               off_C = off_B + up(bbc), off_A = off_C + up(bbc), off_D = off_A + up(bh),
               off_bias = off_D + up(bh), off_init = off_bias + up(bh), off_fin = off_init + up(bst),
               off_cu = off_fin + up(bst), off_y = off_cu + up(bcu), total = off_y + up(by);
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return SSD_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return SSD_ERR_CUDA;
  if (h->io_bytes < total) {
    if (h->io) cudaFree(h->io);
    h->io = nullptr;
    h->io_bytes = 0;
    cudaError_t e = cudaMalloc(&h->io, total);
    if (e != cudaSuccess) {
      h->io = nullptr;
      if (cur != h->device) cudaSetDevice(cur);
      return cuda_rc(e);
    }
    h->io_bytes = total;
  }
  char* base = static_cast<char*>(h->io);
  const size_t bst_call = sizeof(float) * (size_t)ndocs * d.nheads * d.dstate * d.headdim;
  cudaError_t e = cudaSuccess;
  auto h2d = [&](size_t off, const void* src, size_t n) {
    if (src && n && e == cudaSuccess)
      e = cudaMemcpyAsync(base + off, src, n, cudaMemcpyHostToDevice, stream);
  };
  h2d(off_x, x, bx);
  h2d(off_dt, dt, bdt);
  h2d(off_B, B, bbc);
  h2d(off_C, C, bbc);
  h2d(off_A, A, bh);
  h2d(off_D, D, bh);
  h2d(off_bias, dt_bias, bh);
  h2d(off_init, initial_states, bst_call);
  h2d(off_cu, cu_seqlens, cu_seqlens ? sizeof(int32_t) * ((size_t)num_docs + 1) : 0);
  if (e != cudaSuccess) {
    if (cur != h->device) cudaSetDevice(cur);
    return cuda_rc(e);
  }
  rc = ssd_forward(h, base + off_x, base + off_dt, (const float*)(base + off_A), base + off_B,
                   base + off_C, D ? (const float*)(base + off_D) : nullptr,
                   dt_bias ? (const float*)(base + off_bias) : nullptr, chunk_size,
                   initial_states ? (const float*)(base + off_init) : nullptr,
                   cu_seqlens ? (const int32_t*)(base + off_cu) : nullptr, num_docs, base + off_y,
                   final_states ? (float*)(base + off_fin) : nullptr, stream_);
  if (rc == SSD_OK) {
    if (y) e = cudaMemcpyAsync(y, base + off_y, by, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess && final_states)
      e = cudaMemcpyAsync(final_states, base + off_fin, bst_call, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    rc = cuda_rc(e);
  }
  if (cur != h->device) cudaSetDevice(cur);
  return rc;
}

int ssd_get_status(ssd_handle_t h, ssd_stream_t stream_) {
  if (!h) return SSD_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return SSD_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return SSD_ERR_CUDA;
  int v = 0;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && v != 0) e = cudaMemset(h->status, 0, sizeof(int));
  if (cur != h->device) cudaSetDevice(cur);
  if (e != cudaSuccess) return SSD_ERR_CUDA;
  return v;
}

int ssd_debug_line(ssd_handle_t h) {
  if (!h) return SSD_ERR_INVALID_ARG;
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return SSD_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return SSD_ERR_CUDA;
  int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->status + 1, sizeof(int), cudaMemcpyDeviceToHost);
  if (cur != h->device) cudaSetDevice(cur);
  return e == cudaSuccess ? v : SSD_ERR_CUDA;
}

int ssd_debug_build(void) { return SSD_DEBUG_ON; }

int ssd_destroy(ssd_handle_t h) {
  if (!h) return SSD_OK;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != h->device) cudaSetDevice(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  if (h->ws) {
    cudaFreeAsync(h->ws, 0);
    cudaStreamSynchronize(0);
  }
  if (h->io) cudaFree(h->io);
  if (h->status) cudaFree(h->status);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->side) cudaStreamDestroy(h->side);
  if (cur != h->device) cudaSetDevice(cur);
  delete h;
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

const char* ssd_error_string(int code) {
  switch (code) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape or dtype not supported";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA runtime error";
    case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a device-side wait gave up";
    case SSD_ERR_OOM: return "SSD_ERR_OOM: device allocation failed";
    case SSD_ERR_BAD_SEQLENS: return "SSD_ERR_BAD_SEQLENS: cu_seqlens is not a valid partition";
    case SSD_ERR_DEBUG_CHECK:
      return "SSD_ERR_DEBUG_CHECK: a device-side bounds or barrier-phase check failed (debug build)";
    case SSD_ERR_SCRATCH_TOO_SMALL:
      return "SSD_ERR_SCRATCH_TOO_SMALL: the problem needs more scratch than the fixed array";
    default: return "SSD_ERR_UNKNOWN";
  }
}

const char* ssd_version(void) { return "ssd_b200 0.1.0 (sm_100a)"; }

}  // extern "C"
