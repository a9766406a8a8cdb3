// Packed documents: several independent sequences back to back in one token matrix.
//
// The long-context workload of the Motif 3 report (paperglide.net summary, Figure 4a: a packed
// 256K-token sequence of 473 documents) packs documents; each document is its own sequence
// here: rotary positions restart at 0 and attention (causal or sliding window) stays inside
// the document.  These kernels turn cu_seqlens (first row of every document, plus the total)
// into per-token positions and the attention kernel's work units (blocks of ATTN_UNIT_ROWS
// rows of one document), sorted by block index so the longest causal units start first.
#include "gdla_common.cuh"
#include "gdla_internal.h"

namespace gdla {

// position of every token inside its document (binary search over cu_seqlens)
__global__ void varlen_positions_kernel(const int* __restrict__ cu, int n_docs, int total,
                                        int* __restrict__ pos, int* err) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m == 0) {
    bool bad = cu[0] != 0 || cu[n_docs] != total;
    for (int d = 0; d < n_docs && !bad; ++d) bad = cu[d + 1] < cu[d];
    if (bad) atomicCAS(err, 0, SITE_BAD_CU_SEQLENS);
  }
  if (m >= total) return;
  int lo = 0, hi = n_docs - 1;   // last d with cu[d] <= m
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= m) lo = mid; else hi = mid - 1;
  }
  pos[m] = m - cu[lo];
}

// blocks of ATTN_UNIT_ROWS rows of document d; 0 for a document outside [0, total)
__device__ __forceinline__ int doc_blocks(const int* cu, int d, int total, int max_c, int* start,
                                         int* len) {
  *start = cu[d];
  *len = cu[d + 1] - *start;
  if (*start < 0 || *len <= 0 || *start + *len > total) return 0;
  return min((*len + ATTN_UNIT_ROWS - 1) / ATTN_UNIT_ROWS, max_c);
}

// cnt[c] = number of documents with more than c blocks
__global__ void varlen_count_kernel(const int* __restrict__ cu, int n_docs, int total, int* cnt,
                                    int max_c) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= n_docs) return;
  int start, len;
  const int np = doc_blocks(cu, d, total, max_c, &start, &len);
  for (int c = 0; c < np; ++c) atomicAdd(&cnt[c], 1);
}

// offsets for block index c in descending order; one CTA
__global__ void varlen_offsets_kernel(int* cnt, int* fill, int max_c, int* n_units, int max_units,
                                      int* err) {
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int c = max_c - 1; c >= 0; --c) {
      const int k = cnt[c];
      cnt[c] = acc;      // becomes the first slot of block index c
      fill[c] = 0;
      acc += k;
    }
    if (acc > max_units) atomicCAS(err, 0, SITE_BAD_CU_SEQLENS);
    *n_units = min(acc, max_units);
  }
}

__global__ void varlen_fill_kernel(const int* __restrict__ cu, int n_docs, int total, const int* off,
                                   int* fill, int4* units, int max_c, int max_units) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= n_docs) return;
  int start, len;
  const int np = doc_blocks(cu, d, total, max_c, &start, &len);
  for (int c = 0; c < np; ++c) {
    const int slot = off[c] + atomicAdd(&fill[c], 1);
    if (slot < max_units) units[slot] = make_int4(start, len, c, 0);
  }
}

int launch_varlen_schedule(const int* cu_seqlens, int n_docs, int total, int* positions,
                           int4* units, int* n_units, int max_units, int* cnt, int* fill, int max_c,
                           int* err, cudaStream_t st) {
  if (cudaMemsetAsync(cnt, 0, sizeof(int) * max_c, st) != cudaSuccess) return -6;
  varlen_positions_kernel<<<(total + 255) / 256, 256, 0, st>>>(cu_seqlens, n_docs, total, positions, err);
  varlen_count_kernel<<<(n_docs + 255) / 256, 256, 0, st>>>(cu_seqlens, n_docs, total, cnt, max_c);
  varlen_offsets_kernel<<<1, 32, 0, st>>>(cnt, fill, max_c, n_units, max_units, err);
  varlen_fill_kernel<<<(n_docs + 255) / 256, 256, 0, st>>>(cu_seqlens, n_docs, total, cnt, fill, units,
                                                          max_c, max_units);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
