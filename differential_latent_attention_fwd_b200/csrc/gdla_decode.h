// Host-side declarations of the absorbed-form decode kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include "gdla_internal.h"

namespace gdla {

struct DecQParams {
  int B, n_groups, n_signal, n_heads;
  const float* QQ;        // [B, qq_ld] fp32: q^C (head-major) | rotated q^R (head-major)
  int qq_ld, rope_col0;
  const void* W_UKt;      // fp16 [n_groups][128][512]
  void* qt;               // bf16 [B][n_heads][576], fp16 when qt_f16
  int qt_f16;
};

// Upper bound of the decode attention grid (the merge kernel keeps one weight per segment of a
// row in shared memory, and a row has at most one segment per CTA).
constexpr int DEC_MAX_CTAS = 160;

struct DecAttnParams {
  int R;                  // query rows = n_seq x q_len: row r is token r % q_len of sequence r / q_len
  int n_seq, cap, window;
  int q_len;              // new tokens per sequence
  const int* cache_len;   // [n_seq] keys cached before the new tokens
  const void* cache;      // bf16 [n_seq][cap][576], or MXFP8 rows [n_seq][cap][608] (cache_fp8)
  int cache_fp8;
  const void* qt;         // bf16 [R][80][576] (fp16 with an MXFP8 cache)
  float scale_log2;
  int* tstart;            // [R + 1] tile prefix over the rows in list order (dec_sched_kernel)
  int n_ctas;             // grid of the attention kernel (G): slots = G + R - 1
  float* part;            // [slots][80][512] latent accumulators of each segment
  float* ml;              // [slots][80][2]  (running max in log2 units, row sum)
  int* err;               // device error word
};

// Order of the query rows in the attention's work list: token-major, position l = (r % q_len)
// * n_seq + r / q_len for query row r (token r % q_len of sequence r / q_len).  The q_len rows of
// one sequence sit n_seq apart, so with the list split evenly over the CTAs the CTAs serving
// them are about G / q_len apart and reach the same cache tiles at about the same time: the
// second and later reads of a tile hit L2.
__host__ __device__ __forceinline__ int dec_list_pos(int r, int q_len, int n_seq) {
  return q_len > 1 ? (r % q_len) * n_seq + r / q_len : r;
}
__host__ __device__ __forceinline__ int dec_row_of(int l, int q_len, int n_seq) {
  return q_len > 1 ? (l % n_seq) * q_len + l / n_seq : l;
}

// CTAs that take part in the attention's stream-K split of N tiles over a grid of `grid`:
// min(grid, N), rounded down to a multiple of q_len (when that leaves at least q_len) so that
// the q_len token parts of the list start on CTA boundaries.
__host__ __device__ __forceinline__ long long dec_ctas_used(long long N, long long grid, int q_len) {
  long long G = N < grid ? N : grid;
  if (q_len > 1 && G >= q_len) G -= G % q_len;
  return G;
}

struct DecCombParams {
  int B, n_groups, n_signal;   // B = query rows
  int q_len, n_seq;            // (B = q_len * n_seq) for the list order of the rows
  int n_ctas;                  // G of the attention launch
  const int* tstart;           // [B + 1] tile prefix over the rows in list order
  const float* part;           // segment partials, slot c + l for CTA c and list position l
  const float* ml;
  const float* lam;       // [B][n_signal]
  const float* G;         // fp32 gate logits: row b at G + b * g_ld, [n_signal * 128]
  long long g_ld;
  const void* W_bKV;      // bf16 [kv_rank][n_groups * 256]
  void* Dg;               // bf16 [B][n_signal * 128]
};

int launch_absorb_uk(const void* W_bKV, void* W_UKt, int kv_rank, int n_kv, int d_nope, int d_v,
                     cudaStream_t st);
// dst[r][col0 + c] = src[r][c] for r < rows, c < cols (bf16; cols, ld_src, ld_dst, col0
// multiples of 8): concatenation of weight column blocks
int launch_copy_cols(const void* src, long long ld_src, void* dst, long long ld_dst, int col0, int rows,
                     int cols, cudaStream_t st);
int launch_qtilde(const DecQParams& p, KernelCtlHost ctl, cudaStream_t st);
int launch_dec_sched(const DecAttnParams& p, cudaStream_t st);
int launch_dec_attn_tc(const DecAttnParams& p, KernelCtlHost ctl, cudaStream_t st);
int decode_cta_count();
int launch_dec_combine(const DecCombParams& p, KernelCtlHost ctl, cudaStream_t st);

}  // namespace gdla
