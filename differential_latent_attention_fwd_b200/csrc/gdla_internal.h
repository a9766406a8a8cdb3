// Host-side declarations shared by the GDLA translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdla {

enum OutType : int { OUT_F32 = 0, OUT_BF16 = 1, OUT_F16 = 2 };

// Rotary-embedding frequency table, theta^(-2i/d_rope) for i < d_rope/2, in double.
struct RopeTable {
  double inv_freq[32];
  int d_rope;
};

// Epilogue of the projection GEMM C[M, N] = A[M, K] B[K, N].
struct GemmEpi {
  void* C;               // output base (row-major, leading dimension ldc elements)
  long long ldc;
  int out_type;          // OutType
  int M, N;
  int rope_lo, rope_hi;  // columns [rope_lo, rope_hi) (multiples of 64) hold 64-wide rope heads
  int pos_T;             // row position = row % pos_T (used when pos_ptr is null)
  const int* pos_ptr;    // row position = pos_ptr[row / pos_div] + row % pos_div
  int pos_div;           // rows per pos_ptr entry (0 is read as 1)
  int pos_off;           // added to the position (a key prefix of pos_off tokens precedes row 0)
  int row_off;           // row index of output row 0 in the full token matrix (row pieces)
  RopeTable rope;
  // Optional split-K scratch for skinny products (M <= 128): fp32 [splits][M][N].  When set
  // and worthwhile, K is split across CTAs and a reduce kernel applies this epilogue.
  float* splitk;
  long long splitk_floats;
  // internal: set by launch_gemm for the split-K pass (raw fp32 partial tiles)
  float* partial_out;
  int kb_per_split;
  int staged;            // internal: one-tile kernel drains through shared memory (coalesced stores)
  int* err;              // internal: device error word (fp16 outputs out of range are reported)
};

// Number of K splits launch_gemm uses for an M x N x K product (1 = no split).
int gemm_splitk_count(int M, int N, int K);
// Counts a kernel launched by a helper beyond the one its caller counts.
void count_extra_launch();

struct KernelCtlHost {
  int* err;
  unsigned long long limit_ns;
};

// Tensor-map encoding through the driver entry point (no libcuda link dependency).
// Returns 0 on success.  dims/strides as cuTensorMapEncodeTiled: 2-D, innermost first.
int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                 CUtensorMapSwizzle swz);

// C = A * B.  A: [M, K] row-major bf16 (lda elements).  B: bf16, either [K, N] row-major
// (b_kmajor = false, ldb elements) or [N, K] row-major (b_kmajor = true).  K % 64 == 0.
int launch_gemm(const void* A, long long lda, const void* B, long long ldb, bool b_kmajor, int M,
                int N, int K, const GemmEpi& ep, KernelCtlHost ctl, cudaStream_t st);

void fill_rope_table(RopeTable* t, int d_rope, double theta);

// Device error word and current wait bound used by every launch of the library.
int shared_kernel_ctl(KernelCtlHost* out);

// Row-wise epilogue of the down-projection (norms, rotary key, lambda, latent-cache rows).
struct NormParams {
  const float* D1;            // [M, ld1] fp32: x W_a^Q | x W_a^KV | x W^lambda
  int ld1, M;
  int q_rank, kv_rank, n_signal;
  const void* g_q;            // bf16 [q_rank] or null (ones)
  const void* g_kv;           // bf16 [kv_rank] or null
  float eps;
  void* cQ;                   // bf16 [M, q_rank]
  void* latent;               // bf16 [M, kv_rank + 64] or null
  void* kR16;                 // fp16 [M, 64] or null
  float* lam;                 // [M, n_signal]
  int pos_T;                  // prefill: pos = m % pos_T, sequence = m / pos_T
  const int* pos_ptr;         // decode: sequence = m / q_per_seq, pos = pos_ptr[sequence] + m % q_per_seq
  int pos_off;                // added to the position (a key prefix of pos_off tokens precedes row 0)
  int row_off;                // token index of row 0 in the full token matrix (row pieces)
  int q_per_seq;              // new tokens per sequence (0 is read as 1)
  void* cache;                // optional bf16 [n_seq, cache_cap, kv_rank + 64], or MXFP8 rows
  int cache_fp8;              //   [n_seq, cache_cap, 608] when cache_fp8 (norm_rope_row_kernel only)
  long long cache_cap;
  int* err;                   // device error word (bad cache_len is reported here)
  RopeTable rope;
};
int launch_norm_rope(const NormParams& p, cudaStream_t st);

// Fused prefill attention (QK^T, online softmax, PV, differential combine and gate).  One
// work unit = one KV head over ATTN_UNIT_ROWS consecutive query rows of one sequence.
constexpr int ATTN_UNIT_ROWS = 512;
struct AttnParams {
  int B, T, window;           // T = query rows per sequence
  int T_kv;                   // key rows per sequence (= T, or T + q_off with a key prefix)
  int q_off;                  // key position of query row 0 (the length of the key prefix)
  int n_groups;               // KV heads = noise heads
  int n_signal;               // 4 * n_groups
  int rope_col0;              // first q^R column of QQ (n_heads * 128)
  float scale_log2;           // log2(e) / sqrt(d_qk)
  const float* lam;           // [B*T, n_signal]
  const void* G;              // bf16 [B*T, n_signal*128] gate logits
  float* O_noise;             // fp32 scratch, ceil(B*T / 32) * 32 * n_groups * 128 floats: for
                              // row m, group j, column e at
                              // ((m / 32 * n_groups + j) * 32 + e / 4) * 128 + (m % 32) * 4 + e % 4
  void* Dg;                   // bf16 [B*T, n_signal*128]
  // Packed documents (B = 1, T = all tokens): device schedule of work units
  // {first row, document length, block index (rows [512 c, 512 c + 512)), 0}; null for
  // equal-length batches.
  const int4* units;
  const int* n_units;
  int max_units;              // grid bound (units beyond *n_units exit at once)
  // Saved for the backward (null = not written): every head's normalised output H (bf16
  // [B*T, n_heads, d_v]) and log-sum-exp of its scaled scores in log2 units ([B*T, n_heads]).
  void* H_out;
  float* lse_out;
};

// Device schedule of packed documents: per-token positions and the attention work units,
// counting-sorted by block index (heaviest causal units first).  Scratch: cnt/fill [max_c].
int launch_varlen_schedule(const int* cu_seqlens, int n_docs, int total, int* positions,
                           int4* units, int* n_units, int max_units, int* cnt, int* fill, int max_c,
                           int* err, cudaStream_t st);
// Backward of the attention stage (attn_backward.cu).
struct AttnBwdParams {
  int B, T, window, n_signal, n_groups;
  float scale_log2, scale;    // log2(e) / sqrt(d_qk), 1 / sqrt(d_qk)
  const void* QQ;             // fp16 [B*T, n_heads * 192]: q^C of all heads, then rotated q^R
  const void* KV;             // fp16 [B*T, n_groups * 256]: K^C | V per KV head
  const void* kR16;           // fp16 [B*T, 64]: rotated k^R
  const float* lam;           // [B*T, n_signal]
  const void* G;              // bf16 [B*T, n_signal * 128]: gate logits
  const void* H;              // bf16 [B*T, n_heads, 128]: saved per-head outputs
  const float* lse;           // [B*T, n_heads]: saved log2-sum-exp2 of the scaled scores
  const void* d_dg;           // bf16 [B*T, n_signal * 128]: gradient of Dg
  float* d_qq;                // [B*T, n_heads * 192]
  float* d_kv;                // [B*T, n_groups * 256]
  float* d_kr;                // [B*T, 64]
  float* d_lam;               // [B*T, n_signal]
  float* d_G;                 // [B*T, n_signal * 128]
  void* ws;                   // attn_bwd_workspace_bytes(...)
};
size_t attn_bwd_workspace_bytes(long long M, int T, int n_heads, int n_groups);
int launch_attn_bwd(const AttnBwdParams& a, const KernelCtlHost& ctl, cudaStream_t st);

// Rotated k^R of bf16 latent rows (columns kv_rank .. kv_rank + 63) -> fp16 rows of 64.
int launch_latent_to_kr16(const void* latent, int kv_rank, long long rows, void* kR16, int* err,
                          cudaStream_t st);
int launch_attn_prefill(const void* QQ, int qq_ld, const void* KV, const void* kR16,
                        const AttnParams& p, KernelCtlHost ctl, cudaStream_t st);

// MXFP8 latent-cache rows (gdla_fp8.cuh): bf16 rows [rows][576] <-> stored rows [rows][608]
int launch_mxfp8_quantize(const void* in, long long rows, void* out, cudaStream_t st);
int launch_mxfp8_dequantize(const void* in, long long rows, void* out, cudaStream_t st);

}  // namespace gdla
