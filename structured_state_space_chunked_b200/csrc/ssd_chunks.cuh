// ssd_chunks.cuh -- the chunk table lookup shared by the chunk-parallel kernels
// (the CUDA-core forward and the backward).  Chunks of Q tokens never straddle a
// document; packed documents take their chunk table from the workspace, which
// the varlen_table kernel fills on the device.
#pragma once

#include "ssd_internal.h"

namespace ssd {

struct ChunkInfo {
  int doc;
  int c;           // chunk index within the document
  int64_t start;   // first token
  int len;         // tokens in the chunk (1..Q)
};

// Chunk k of the problem; false for chunk slots past the end (varlen upper bound).
__device__ __forceinline__ bool chunk_info(const Geom& g, const int32_t* cu,
                                           const SimtWorkspace& ws, int64_t k, ChunkInfo* ci) {
  if (!g.varlen) {
    const int64_t nc = (g.seqlen + g.Q - 1) / g.Q;
    if (nc == 0 || k >= (int64_t)g.ndocs * nc) return false;
    ci->doc = (int)(k / nc);
    ci->c = (int)(k % nc);
    ci->start = (int64_t)ci->doc * g.seqlen + (int64_t)ci->c * g.Q;
    ci->len = (int)min((int64_t)g.Q, g.seqlen - (int64_t)ci->c * g.Q);
    return true;
  }
  if (!ws.total_chunks[1] || k >= ws.total_chunks[0]) return false;
  const int d = ws.chunk_doc[k];
  ci->doc = d;
  ci->c = (int)(k - ws.doc_first[d]);
  ci->start = (int64_t)cu[d] + (int64_t)ci->c * g.Q;
  ci->len = (int)min((int64_t)g.Q, (int64_t)cu[d + 1] - ci->start);
  return true;
}

// Number of chunks of document d (the chunks of a document are consecutive).
__device__ __forceinline__ int64_t doc_chunks(const Geom& g, const SimtWorkspace& ws, int d,
                                              int64_t* first) {
  if (g.varlen) {
    *first = ws.doc_first[d];
    return ws.doc_first[d + 1] - *first;
  }
  const int64_t nc = (g.seqlen + g.Q - 1) / g.Q;
  *first = (int64_t)d * nc;
  return nc;
}

}  // namespace ssd
