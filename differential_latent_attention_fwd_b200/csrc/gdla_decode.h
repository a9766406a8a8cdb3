// Host-side declarations of the absorbed-form decode kernels (internal).
#pragma once

#include <cuda_runtime.h>

#include "gdla_internal.h"

namespace gdla {

struct DecQParams {
  int B, n_groups, n_signal, n_heads;
  const float* QQ;        // [B, qq_ld] fp32: q^C (head-major) | rotated q^R (head-major)
  int qq_ld, rope_col0;
  const void* W_UKt;      // bf16 [n_groups][128][512]
  void* qt;               // bf16 [B][n_heads][576]
};

struct DecAttnParams {
  int B, cap, window, n_split;   // B = query rows = sequences x q_len
  int q_len;              // new tokens per sequence: row r is token r % q_len of sequence r / q_len
  const int* cache_len;   // [sequences] keys cached before the new tokens
  const void* cache;      // bf16 [B][cap][576]
  const void* qt;         // bf16 [B][80][576]
  float scale_log2;
  float* part;            // [B][n_split][80][512] latent accumulators
  float* ml;              // [B][n_split][80][2]  (running max in log2 units, row sum)
  int* err;               // device error word
};

struct DecCombParams {
  int B, n_groups, n_signal, n_split;
  const float* part;
  const float* ml;
  const float* lam;       // [B][n_signal]
  const void* G;          // bf16 [B][n_signal * 128]
  const void* W_bKV;      // bf16 [kv_rank][n_groups * 256]
  void* Dg;               // bf16 [B][n_signal * 128]
};

int launch_absorb_uk(const void* W_bKV, void* W_UKt, int kv_rank, int n_kv, int d_nope, int d_v,
                     cudaStream_t st);
int launch_qtilde(const DecQParams& p, cudaStream_t st);
int launch_dec_attn_tc(const DecAttnParams& p, KernelCtlHost ctl, cudaStream_t st);
int decode_split_count(int B, int cap, int window);
int launch_dec_combine(const DecCombParams& p, cudaStream_t st);

}  // namespace gdla
