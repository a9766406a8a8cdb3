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
// a call never accumulates two heads into the same dK / dV rows).  Queries and keys are first
// gathered into 192-wide rows q = [q^C | q^R], k_j = [K^C_j | k^R], so that the scores, dq and
// dk are one contraction each; P and dS' are formed by one elementwise pass over the fp32
// scores.  The key range of a block is the causal (or window) range of its rows.
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

// P = 2^(S scale_log2 - LSE2) (fp16, for dV = P^T dH) and dS' = P (dP - Delta) / sqrt(d_qk)
// (fp16, for dq and dk) on the visible keys, 0 elsewhere.  Grid (column quads, query row,
// group); a thread forms four consecutive columns.
__global__ void bwd_p_ds_kernel(const float* __restrict__ S, const float* __restrict__ dP,
                                const float* __restrict__ lse, const float* __restrict__ delta, BwdBlock b,
                                __half* __restrict__ P, __half* __restrict__ dS) {
  const int c0 = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (c0 >= b.ldk) return;
  const int r = blockIdx.y, j = blockIdx.z;
  const int q = b.q0 + r;
  const int nH = b.n_signal + b.n_groups;
  const int h = head_of(b.slot, j, b.n_signal, b.n_signal / b.n_groups);
  const long long hr = (b.row0 + r) * nH + h;
  const float l2 = lse[hr], dl = delta[hr];
  const long long i = ((long long)j * b.nq + r) * b.ldk + c0;
  const float4 s4 = *reinterpret_cast<const float4*>(S + i);
  const float4 d4 = *reinterpret_cast<const float4*>(dP + i);
  const float sv[4] = {s4.x, s4.y, s4.z, s4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
  __half pv[4], gv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = c0 + e, k = b.k_lo + c;
    const bool vis = c < b.nk && k <= q && (b.window <= 0 || k > q - b.window);
    const float p = vis ? exp2f(sv[e] * b.scale_log2 - l2) : 0.f;
    pv[e] = __float2half_rn(p);
    gv[e] = __float2half_rn(p * (dv[e] - dl) * b.scale);
  }
  *reinterpret_cast<uint2*>(P + i) = *reinterpret_cast<const uint2*>(pv);
  *reinterpret_cast<uint2*>(dS + i) = *reinterpret_cast<const uint2*>(gv);
}

// q rows of every head as [q^C | rotated q^R] (192 halves): Q192[m][h] from the QQ row layout
// (q^C of all heads, then q^R of all heads).  One thread per 16-byte chunk.
__global__ void bwd_gather_q_kernel(const __half* __restrict__ QQ, long long M, int nH, __half* __restrict__ Q192) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= M * nH * 24) return;
  const int ch = int(t % 24);
  const long long mh = t / 24;
  const long long m = mh / nH;
  const int h = int(mh % nH);
  const __half* src = ch < 16 ? QQ + m * nH * 192 + (long long)h * 128 + ch * 8
                              : QQ + m * nH * 192 + (long long)nH * 128 + (long long)h * 64 + (ch - 16) * 8;
  *reinterpret_cast<uint4*>(Q192 + mh * 192 + ch * 8) = *reinterpret_cast<const uint4*>(src);
}

// key rows of every KV group as [K^C_j | rotated k^R] (192 halves).
__global__ void bwd_gather_k_kernel(const __half* __restrict__ KV, const __half* __restrict__ kR, long long M,
                                    int n_groups, __half* __restrict__ K192) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= M * n_groups * 24) return;
  const int ch = int(t % 24);
  const long long mj = t / 24;
  const long long m = mj / n_groups;
  const int j = int(mj % n_groups);
  const __half* src = ch < 16 ? KV + m * n_groups * 256 + (long long)j * 256 + ch * 8 : kR + m * 64 + (ch - 16) * 8;
  *reinterpret_cast<uint4*>(K192 + mj * 192 + ch * 8) = *reinterpret_cast<const uint4*>(src);
}

// dq of a block's rows: [dq^C | dq^R] per head (fp32) -> the QQ column layout of d_qq.
__global__ void bwd_scatter_q_kernel(const float* __restrict__ dQ192, long long row0, int nq, int nH,
                                     float* __restrict__ d_qq) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)nq * nH * 48) return;
  const int ch = int(t % 48);
  const long long rh = t / 48;
  const long long r = rh / nH;
  const int h = int(rh % nH);
  float* dst = d_qq + (row0 + r) * nH * 192 +
               (ch < 32 ? (long long)h * 128 + ch * 4 : (long long)nH * 128 + (long long)h * 64 + (ch - 32) * 4);
  *reinterpret_cast<float4*>(dst) = *reinterpret_cast<const float4*>(dQ192 + rh * 192 + ch * 4);
}

// dK^C_j -> d_kv (its K^C columns), and dk^R = sum over the groups of their k^R parts.
__global__ void bwd_finish_k_kernel(const float* __restrict__ dK192, long long M, int n_groups,
                                    float* __restrict__ d_kv, float* __restrict__ d_kr) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nc = (long long)n_groups * 32 + 16;   // float4 chunks per row: K^C parts, then dk^R
  if (t >= M * nc) return;
  const long long m = t / nc;
  const int ch = int(t % nc);
  if (ch < n_groups * 32) {
    const int j = ch / 32, c = (ch % 32) * 4;
    *reinterpret_cast<float4*>(d_kv + m * n_groups * 256 + (long long)j * 256 + c) =
        *reinterpret_cast<const float4*>(dK192 + (m * n_groups + j) * 192 + c);
  } else {
    const int c = 128 + (ch - n_groups * 32) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < n_groups; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(dK192 + (m * n_groups + j) * 192 + c);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *reinterpret_cast<float4*>(d_kr + m * 64 + (c - 128)) = acc;
  }
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
  const size_t sbuf = (size_t)n_groups * ATTN_BWD_BQ * ldk;
  return al(M * n_heads * 128 * 2) + al(M * n_heads * 4) + al(M * n_heads * 192 * 2) +
         al(M * n_groups * 192 * 2) + al(M * n_groups * 192 * 4) + al((size_t)ATTN_BWD_BQ * n_heads * 192 * 4) +
         2 * al(sbuf * 4) + 2 * al(sbuf * 2) + al(32u << 20);
}

int launch_attn_bwd(const AttnBwdParams& a, cudaStream_t st) {
  cublasHandle_t h = blas_handle();
  if (!h) return -6;
  const long long M = (long long)a.B * a.T;
  const int nH = a.n_signal + a.n_groups, gsz = a.n_signal / a.n_groups, ng = a.n_groups;
  const int ldk = (a.T + 7) / 8 * 8;
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  uint8_t* w = static_cast<uint8_t*>(a.ws);
  __half* dO = reinterpret_cast<__half*>(w); w += al(M * nH * 128 * 2);
  float* delta = reinterpret_cast<float*>(w); w += al(M * nH * 4);
  __half* Q192 = reinterpret_cast<__half*>(w); w += al(M * nH * 192 * 2);
  __half* K192 = reinterpret_cast<__half*>(w); w += al(M * ng * 192 * 2);
  float* dK192 = reinterpret_cast<float*>(w); w += al(M * ng * 192 * 4);
  float* dQ192 = reinterpret_cast<float*>(w); w += al((size_t)ATTN_BWD_BQ * nH * 192 * 4);
  const size_t sbuf = (size_t)ng * ATTN_BWD_BQ * ldk;
  float* S = reinterpret_cast<float*>(w); w += al(sbuf * 4);
  float* dP = reinterpret_cast<float*>(w); w += al(sbuf * 4);
  __half* P = reinterpret_cast<__half*>(w); w += al(sbuf * 2);
  __half* dS = reinterpret_cast<__half*>(w); w += al(sbuf * 2);
  void* blas_ws = w;
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS ||
      cublasSetWorkspace(h, blas_ws, 32u << 20) != CUBLAS_STATUS_SUCCESS)
    return -6;

  const __half* QQ = static_cast<const __half*>(a.QQ);
  const __half* KV = static_cast<const __half*>(a.KV);
  const __half* KR = static_cast<const __half*>(a.kR16);
  {
    const long long warps = M * ng;
    bwd_pre_kernel<<<unsigned((warps + 7) / 8), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.d_dg), static_cast<const __nv_bfloat16*>(a.G), a.lam,
        static_cast<const __nv_bfloat16*>(a.H), M, ng, a.n_signal, dO, delta, a.d_lam, a.d_G);
    const long long nq_ch = M * nH * 24, nk_ch = M * ng * 24;
    bwd_gather_q_kernel<<<unsigned((nq_ch + 255) / 256), 256, 0, st>>>(QQ, M, nH, Q192);
    bwd_gather_k_kernel<<<unsigned((nk_ch + 255) / 256), 256, 0, st>>>(KV, KR, M, ng, K192);
    if (cudaPeekAtLastError() != cudaSuccess) return -4;
  }
  // dV accumulates into the V columns of d_kv; the K^C columns are written at the end
  if (cudaMemsetAsync(a.d_kv, 0, (size_t)M * ng * 256 * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dK192, 0, (size_t)M * ng * 192 * 4, st) != cudaSuccess)
    return -6;

  const int kv_ld = ng * 256, q_ld = nH * 192, k_ld = ng * 192;
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
      bk.window = a.window; bk.n_signal = a.n_signal; bk.n_groups = ng;
      bk.scale_log2 = a.scale_log2; bk.scale = a.scale;
      const long long krow = (long long)b * a.T + bk.k_lo;     // token row of key 0
      const long long sS = (long long)bk.nq * bk.ldk;          // batch stride of the score buffers
      const __half* Kb = K192 + krow * k_ld;
      const __half* Vb = KV + krow * kv_ld + 128;
      for (int i = 0; i <= gsz; ++i) {
        bk.slot = i;
        // head of group j at slot i: i = 0 noise (n_signal + j, stride 1 head), else 4 j + i - 1 (stride 4)
        const int h0 = i == 0 ? a.n_signal : i - 1;
        const int hs = i == 0 ? 1 : gsz;
        const __half* Qs = Q192 + bk.row0 * q_ld + (long long)h0 * 192;
        const __half* dOh = dO + bk.row0 * nH * 128 + (long long)h0 * 128;
        bool ok = true;
        // S = [q^C | q^R] [K^C | k^R]^T
        ok = ok && gemm_rm(h, false, true, bk.nq, bk.nk, 192, 1.f, Qs, F16, q_ld, (long long)hs * 192,
                           Kb, F16, k_ld, 192, 0.f, S, F32, bk.ldk, sS, ng);
        // dP = dH V^T
        ok = ok && gemm_rm(h, false, true, bk.nq, bk.nk, 128, 1.f, dOh, F16, nH * 128, (long long)hs * 128,
                           Vb, F16, kv_ld, 256, 0.f, dP, F32, bk.ldk, sS, ng);
        if (!ok) return -6;
        {
          const dim3 grid(unsigned((bk.ldk / 4 + 127) / 128), unsigned(bk.nq), unsigned(ng));
          bwd_p_ds_kernel<<<grid, 128, 0, st>>>(S, dP, a.lse, delta, bk, P, dS);
          if (cudaPeekAtLastError() != cudaSuccess) return -4;
        }
        // dq = dS' [K^C | k^R];  d[K^C | k^R] += dS'^T [q^C | q^R];  dV += P^T dH
        ok = ok && gemm_rm(h, false, false, bk.nq, 192, bk.nk, 1.f, dS, F16, bk.ldk, sS, Kb, F16, k_ld, 192,
                           0.f, dQ192 + (long long)h0 * 192, F32, q_ld, (long long)hs * 192, ng);
        ok = ok && gemm_rm(h, true, false, bk.nk, 192, bk.nq, 1.f, dS, F16, bk.ldk, sS, Qs, F16, q_ld,
                           (long long)hs * 192, 1.f, dK192 + krow * k_ld, F32, k_ld, 192, ng);
        ok = ok && gemm_rm(h, true, false, bk.nk, 128, bk.nq, 1.f, P, F16, bk.ldk, sS, dOh, F16, nH * 128,
                           (long long)hs * 128, 1.f, a.d_kv + krow * kv_ld + 128, F32, kv_ld, 256, ng);
        if (!ok) return -6;
      }
      const long long n_ch = (long long)bk.nq * nH * 48;
      bwd_scatter_q_kernel<<<unsigned((n_ch + 255) / 256), 256, 0, st>>>(dQ192, bk.row0, bk.nq, nH, a.d_qq);
      if (cudaPeekAtLastError() != cudaSuccess) return -4;
    }
  }
  const long long n_fin = M * ((long long)ng * 32 + 16);
  bwd_finish_k_kernel<<<unsigned((n_fin + 255) / 256), 256, 0, st>>>(dK192, M, ng, a.d_kv, a.d_kr);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
