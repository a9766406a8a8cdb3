// Backward of the GDLA attention stage (picx.dev "Motif 3" summary, section 2.2: per-head
// softmax attention, D = H_S - lambda Repeat_g(H_N), sigmoid(G) gate), given the gradient of
// its output Dg and the per-head outputs H and log-sum-exp saved by the forward.
//
// By the chain rule, with g = sigmoid(G) and D = H_S - lambda H_N:
//   dG = dDg g (1 - g) D;  dH_S = dDg g;  dlambda_s = -sum_c dH_S[c] H_N(s)[c];
//   dH_N(n) = -sum_{s -> n} lambda_s dH_S;  Delta_h = sum_c dH_h[c] H_h[c];
// and for every head, with P = 2^(s log2e / sqrt(192) - LSE2) recomputed from the scores:
//   dV += P^T dH,  dP = dH V^T,  dS' = P (dP - Delta) / sqrt(192),
//   dq = dS' [K^C ; k^R],  d[K^C ; k^R] += dS'^T [q^C ; q^R].
// The contractions run as strided-batched GEMMs (cuBLAS, fp16 operands, fp32 accumulate) over
// one query block of one sequence and, per call, one head of each of the 16 KV groups (so that
// a call never accumulates two heads into the same dK^C / dV rows); P and dS' are formed by the
// kernels below.  The key range of a block is the causal (or window) range of its rows.
#include <cublas_v2.h>

#include <mutex>

#include "gdla_common.cuh"
#include "gdla_internal.h"

namespace gdla {

// ---- per (row m, KV group j): dDg -> dH of the group's four signal heads and its noise head,
// Delta of all five, dlambda, dG.  One warp; lane owns columns 4 lane .. 4 lane + 3.
__global__ void bwd_pre_kernel(const __nv_bfloat16* __restrict__ dDg, const __nv_bfloat16* __restrict__ G,
                               const float* __restrict__ lam, const __nv_bfloat16* __restrict__ H,
                               long long M, int n_groups, int n_signal, __half* __restrict__ dO,
                               float* __restrict__ delta, float* __restrict__ dlam, float* __restrict__ dG) {
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= M * n_groups) return;
  const long long m = wid / n_groups;
  const int j = int(wid % n_groups);
  const int nH = n_signal + n_groups;
  const int g = n_signal / n_groups;
  const int c0 = 4 * lane;
  float hn[4], dhn[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const __nv_bfloat16* hr = H + (m * nH + n_signal + j) * 128 + c0;
#pragma unroll
    for (int e = 0; e < 4; ++e) hn[e] = __bfloat162float(hr[e]);
  }
  for (int k = 0; k < g; ++k) {
    const int s = g * j + k;
    const long long row = m * n_signal + s;
    const float l = lam[row];
    float hs[4], dh[4], acc_delta = 0.f, acc_dl = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float gv = 1.0f / (1.0f + __expf(-__bfloat162float(G[row * 128 + c0 + e])));
      const float dd = __bfloat162float(dDg[row * 128 + c0 + e]);
      hs[e] = __bfloat162float(H[(m * nH + s) * 128 + c0 + e]);
      dG[row * 128 + c0 + e] = dd * gv * (1.0f - gv) * (hs[e] - l * hn[e]);
      dh[e] = dd * gv;
      acc_delta += dh[e] * hs[e];
      acc_dl -= dh[e] * hn[e];
      dhn[e] -= l * dh[e];
      dO[(m * nH + s) * 128 + c0 + e] = __float2half_rn(dh[e]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      acc_delta += __shfl_xor_sync(0xffffffffu, acc_delta, o);
      acc_dl += __shfl_xor_sync(0xffffffffu, acc_dl, o);
    }
    if (lane == 0) {
      delta[m * nH + s] = acc_delta;
      dlam[row] = acc_dl;
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    dO[(m * nH + n_signal + j) * 128 + c0 + e] = __float2half_rn(dhn[e]);
    acc += dhn[e] * hn[e];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) delta[m * nH + n_signal + j] = acc;
}

// Head of KV group j at slot i of the group: 0 = the noise head, 1..g = the signal heads.
__device__ __forceinline__ int head_of(int i, int j, int n_signal, int g) {
  return i == 0 ? n_signal + j : g * j + i - 1;
}

struct BwdBlock {
  long long row0;       // token row of query 0 of the block (sequence start + q0)
  int q0, nq;           // first query position of the block, number of queries
  int k_lo, nk, ldk;    // first key position, number of keys, row stride of the score buffers
  int window, n_signal, n_groups, slot;
  float scale_log2;     // log2(e) / sqrt(d_qk)
  float scale;          // 1 / sqrt(d_qk)
};

// P = 2^(S scale_log2 - LSE2) on the visible keys, 0 elsewhere (fp16, for dV = P^T dH).
__global__ void bwd_p_kernel(const float* __restrict__ S, const float* __restrict__ lse, BwdBlock b,
                             __half* __restrict__ P) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long per = (long long)b.nq * b.ldk;
  if (i >= per * b.n_groups) return;
  const int j = int(i / per);
  const int r = int((i % per) / b.ldk), c = int(i % b.ldk);
  const int q = b.q0 + r, k = b.k_lo + c;
  const int nH = b.n_signal + b.n_groups;
  const int h = head_of(b.slot, j, b.n_signal, b.n_signal / b.n_groups);
  const bool vis = c < b.nk && k <= q && (b.window <= 0 || k > q - b.window);
  float p = 0.f;
  if (vis) p = exp2f(S[i] * b.scale_log2 - lse[(b.row0 + r) * nH + h]);
  P[i] = __float2half_rn(p);
}

// dS' = P (dP - Delta) / sqrt(d_qk), P recomputed from the fp32 scores.
__global__ void bwd_ds_kernel(const float* __restrict__ S, const float* __restrict__ dP,
                              const float* __restrict__ lse, const float* __restrict__ delta, BwdBlock b,
                              __half* __restrict__ dS) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long per = (long long)b.nq * b.ldk;
  if (i >= per * b.n_groups) return;
  const int j = int(i / per);
  const int r = int((i % per) / b.ldk), c = int(i % b.ldk);
  const int q = b.q0 + r, k = b.k_lo + c;
  const int nH = b.n_signal + b.n_groups;
  const int h = head_of(b.slot, j, b.n_signal, b.n_signal / b.n_groups);
  const bool vis = c < b.nk && k <= q && (b.window <= 0 || k > q - b.window);
  float v = 0.f;
  if (vis) {
    const long long hr = (b.row0 + r) * nH + h;
    const float p = exp2f(S[i] * b.scale_log2 - lse[hr]);
    v = p * (dP[i] - delta[hr]) * b.scale;
  }
  dS[i] = __float2half_rn(v);
}

__global__ void bwd_sum_kr_kernel(const float* __restrict__ part, long long M, int n_groups, float* __restrict__ dkR) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * 64) return;
  float acc = 0.f;
  for (int j = 0; j < n_groups; ++j) acc += part[(long long)j * M * 64 + i];
  dkR[i] = acc;
}

// ---- cuBLAS: one handle per device, created on first use and kept.
namespace {
std::mutex g_blas_mu;
cublasHandle_t g_blas[64] = {};
}  // namespace

static cublasHandle_t blas_handle() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_blas_mu);
  if (!g_blas[dev] && cublasCreate(&g_blas[dev]) != CUBLAS_STATUS_SUCCESS) g_blas[dev] = nullptr;
  return g_blas[dev];
}

// Row-major C[M x N] = alpha op(A) op(B) + beta C, strided batch of `batch` (column-major
// cuBLAS on the transposed problem: C^T = op(B)^T op(A)^T).
static bool gemm_rm(cublasHandle_t h, bool ta, bool tb, int M, int N, int K, float alpha,
                    const void* A, cudaDataType ta_type, int lda, long long sa,
                    const void* B, cudaDataType tb_type, int ldb, long long sb, float beta,
                    void* C, cudaDataType tc_type, int ldc, long long sc, int batch) {
  return cublasGemmStridedBatchedEx(h, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N,
                                    N, M, K, &alpha, B, tb_type, ldb, sb, A, ta_type, lda, sa, &beta,
                                    C, tc_type, ldc, sc, batch, CUBLAS_COMPUTE_32F,
                                    CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
}

size_t attn_bwd_workspace_bytes(long long M, int T, int n_heads, int n_groups) {
  const long long ldk = ((long long)T + 7) / 8 * 8;
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  return al(M * n_heads * 128 * 2) + al(M * n_heads * 4) + 2 * al((size_t)n_groups * ATTN_BWD_BQ * ldk * 4) +
         2 * al((size_t)n_groups * ATTN_BWD_BQ * ldk * 2) + al((size_t)n_groups * M * 64 * 4) + al(32u << 20);
}

int launch_attn_bwd(const AttnBwdParams& a, cudaStream_t st) {
  cublasHandle_t h = blas_handle();
  if (!h) return -6;
  const long long M = (long long)a.B * a.T;
  const int nH = a.n_signal + a.n_groups, gsz = a.n_signal / a.n_groups;
  const int ldk = (a.T + 7) / 8 * 8;
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  uint8_t* w = static_cast<uint8_t*>(a.ws);
  __half* dO = reinterpret_cast<__half*>(w); w += al(M * nH * 128 * 2);
  float* delta = reinterpret_cast<float*>(w); w += al(M * nH * 4);
  const size_t sbuf = (size_t)a.n_groups * ATTN_BWD_BQ * ldk;
  float* S = reinterpret_cast<float*>(w); w += al(sbuf * 4);
  float* dP = reinterpret_cast<float*>(w); w += al(sbuf * 4);
  __half* P = reinterpret_cast<__half*>(w); w += al(sbuf * 2);
  __half* dS = reinterpret_cast<__half*>(w); w += al(sbuf * 2);
  float* kr_part = reinterpret_cast<float*>(w); w += al((size_t)a.n_groups * M * 64 * 4);
  void* blas_ws = w;
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS ||
      cublasSetWorkspace(h, blas_ws, 32u << 20) != CUBLAS_STATUS_SUCCESS)
    return -6;

  {
    const long long warps = M * a.n_groups;
    bwd_pre_kernel<<<unsigned((warps + 7) / 8), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.d_dg), static_cast<const __nv_bfloat16*>(a.G), a.lam,
        static_cast<const __nv_bfloat16*>(a.H), M, a.n_groups, a.n_signal, dO, delta, a.d_lam, a.d_G);
    if (cudaPeekAtLastError() != cudaSuccess) return -4;
  }
  if (cudaMemsetAsync(a.d_kv, 0, (size_t)M * a.n_groups * 256 * 4, st) != cudaSuccess ||
      cudaMemsetAsync(kr_part, 0, (size_t)a.n_groups * M * 64 * 4, st) != cudaSuccess)
    return -6;

  const int qq_ld = nH * 192, kv_ld = a.n_groups * 256;
  const int rope0 = nH * 128;   // first q^R column of a QQ row
  const __half* QQ = static_cast<const __half*>(a.QQ);
  const __half* KV = static_cast<const __half*>(a.KV);
  const __half* KR = static_cast<const __half*>(a.kR16);
  float* dQQ = a.d_qq;
  float* dKV = a.d_kv;
  const auto F16 = CUDA_R_16F, F32 = CUDA_R_32F;
  for (int b = 0; b < a.B; ++b) {
    for (int q0 = 0; q0 < a.T; q0 += ATTN_BWD_BQ) {
      BwdBlock bk{};
      bk.nq = a.T - q0 < ATTN_BWD_BQ ? a.T - q0 : ATTN_BWD_BQ;
      bk.q0 = q0;
      bk.row0 = (long long)b * a.T + q0;
      bk.k_lo = a.window > 0 ? (q0 - a.window + 1 > 0 ? q0 - a.window + 1 : 0) : 0;
      bk.nk = q0 + bk.nq - bk.k_lo;
      bk.ldk = (bk.nk + 7) / 8 * 8;
      bk.window = a.window; bk.n_signal = a.n_signal; bk.n_groups = a.n_groups;
      bk.scale_log2 = a.scale_log2; bk.scale = a.scale;
      const long long krow = (long long)b * a.T + bk.k_lo;     // token row of key 0
      const long long sS = (long long)bk.nq * bk.ldk;          // batch stride of the score buffers
      const long long n_el = sS * a.n_groups;
      for (int i = 0; i <= gsz; ++i) {
        bk.slot = i;
        // head of group j at slot i: i = 0 noise (n_signal + j, stride 1 head), else 4 j + i - 1 (stride 4)
        const int h0 = i == 0 ? a.n_signal : i - 1;
        const int hs = i == 0 ? 1 : gsz;
        const __half* qC = QQ + bk.row0 * qq_ld + (long long)h0 * 128;
        const __half* qR = QQ + bk.row0 * qq_ld + rope0 + (long long)h0 * 64;
        const __half* KC = KV + krow * kv_ld;
        const __half* Vv = KV + krow * kv_ld + 128;
        const __half* kR = KR + krow * 64;
        const __half* dOh = dO + bk.row0 * nH * 128 + (long long)h0 * 128;
        bool ok = true;
        // S = q^C K^C^T + q^R k^R^T
        ok = ok && gemm_rm(h, false, true, bk.nq, bk.nk, 128, 1.f, qC, F16, qq_ld, (long long)hs * 128,
                           KC, F16, kv_ld, 256, 0.f, S, F32, bk.ldk, sS, a.n_groups);
        ok = ok && gemm_rm(h, false, true, bk.nq, bk.nk, 64, 1.f, qR, F16, qq_ld, (long long)hs * 64,
                           kR, F16, 64, 0, 1.f, S, F32, bk.ldk, sS, a.n_groups);
        // dP = dH V^T
        ok = ok && gemm_rm(h, false, true, bk.nq, bk.nk, 128, 1.f, dOh, F16, nH * 128, (long long)hs * 128,
                           Vv, F16, kv_ld, 256, 0.f, dP, F32, bk.ldk, sS, a.n_groups);
        if (!ok) return -6;
        const unsigned blocks = unsigned((n_el + 255) / 256);
        bwd_p_kernel<<<blocks, 256, 0, st>>>(S, a.lse, bk, P);
        bwd_ds_kernel<<<blocks, 256, 0, st>>>(S, dP, a.lse, delta, bk, dS);
        if (cudaPeekAtLastError() != cudaSuccess) return -4;
        float* dqC = dQQ + bk.row0 * qq_ld + (long long)h0 * 128;
        float* dqR = dQQ + bk.row0 * qq_ld + rope0 + (long long)h0 * 64;
        // dq = dS' [K^C ; k^R]
        ok = ok && gemm_rm(h, false, false, bk.nq, 128, bk.nk, 1.f, dS, F16, bk.ldk, sS, KC, F16, kv_ld, 256,
                           0.f, dqC, F32, qq_ld, (long long)hs * 128, a.n_groups);
        ok = ok && gemm_rm(h, false, false, bk.nq, 64, bk.nk, 1.f, dS, F16, bk.ldk, sS, kR, F16, 64, 0,
                           0.f, dqR, F32, qq_ld, (long long)hs * 64, a.n_groups);
        // d[K^C ; k^R] += dS'^T [q^C ; q^R];  dV += P^T dH
        ok = ok && gemm_rm(h, true, false, bk.nk, 128, bk.nq, 1.f, dS, F16, bk.ldk, sS, qC, F16, qq_ld,
                           (long long)hs * 128, 1.f, dKV + krow * kv_ld, F32, kv_ld, 256, a.n_groups);
        ok = ok && gemm_rm(h, true, false, bk.nk, 64, bk.nq, 1.f, dS, F16, bk.ldk, sS, qR, F16, qq_ld,
                           (long long)hs * 64, 1.f, kr_part + krow * 64, F32, 64, M * 64, a.n_groups);
        ok = ok && gemm_rm(h, true, false, bk.nk, 128, bk.nq, 1.f, P, F16, bk.ldk, sS, dOh, F16, nH * 128,
                           (long long)hs * 128, 1.f, dKV + krow * kv_ld + 128, F32, kv_ld, 256, a.n_groups);
        if (!ok) return -6;
      }
    }
  }
  bwd_sum_kr_kernel<<<unsigned((M * 64 + 255) / 256), 256, 0, st>>>(kr_part, M, a.n_groups, a.d_kr);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
