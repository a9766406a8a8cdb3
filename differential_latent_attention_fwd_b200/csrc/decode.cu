// Weight-absorbed GDLA decode: one new token per sequence attends over its latent cache.
//
// The paperglide.net "Model Architecture" section notes that MLA keeps one low-rank latent
// per token and rebuilds per-head keys/values only inside the attention computation.  With
// W_UK_j / W_UV_j the K^C / V column blocks of W_b^KV for KV head j (picx.dev summary,
// section 2.2, [K^C; V] = Reshape_heads(c_bar W_b^KV)) the decode step regroups the products:
//   q~_h   = W_UK_j q^C_h                          (query moved into the 512-wide latent space)
//   s_h,p  = (q~_h . c_bar_p + q^R_h . k^R_p) / sqrt(192)
//   l_h    = sum_p softmax_p(s_h) c_bar_p          (attention output, still latent)
//   D_s    = (l_s - lambda_s l_noise(j)) W_UV_j    (differential combine before the up-projection)
//   Dg_s   = sigmoid(G_s) (.) D_s
// so every cached byte (c_bar | k^R, 1152 bytes per position) is read once for all 80 heads.
//
// Kernels here: W_UK transpose (weight absorption), q~ formation, split-K latent attention
// with per-split partial (max, sum, latent accumulator), and the split merge + combine + gate.
#include "gdla_common.cuh"
#include "gdla_internal.h"
#include "gdla_decode.h"

namespace gdla {

// W_UKt[j][c][l] = W_bKV[l][j * (d_nope + d_v) + c]
__global__ void absorb_uk_kernel(const __nv_bfloat16* __restrict__ W_bKV, __nv_bfloat16* __restrict__ W_UKt,
                                 int kv_rank, int n_kv, int d_nope, int d_v) {
  const long long total = (long long)n_kv * d_nope * kv_rank;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int l = int(i % kv_rank);
    const int c = int((i / kv_rank) % d_nope);
    const int j = int(i / ((long long)kv_rank * d_nope));
    W_UKt[i] = W_bKV[(long long)l * n_kv * (d_nope + d_v) + j * (d_nope + d_v) + c];
  }
}

int launch_absorb_uk(const void* W_bKV, void* W_UKt, int kv_rank, int n_kv, int d_nope, int d_v,
                     cudaStream_t st) {
  absorb_uk_kernel<<<1024, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W_bKV),
                                         static_cast<__nv_bfloat16*>(W_UKt), kv_rank, n_kv, d_nope, d_v);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// q~ rows: qt[b][h][0..511] = W_UK_j q^C_h, qt[b][h][512..575] = rotated q^R_h (bf16).
// One CTA per (sequence b, KV head j) serves the group's g + 1 heads.
__global__ void __launch_bounds__(256) qtilde_kernel(DecQParams p) {
  const int b = blockIdx.x, j = blockIdx.y;
  __shared__ float qc[5][128];
  const int heads[5] = {p.n_signal + j, 4 * j, 4 * j + 1, 4 * j + 2, 4 * j + 3};
  for (int i = threadIdx.x; i < 5 * 128; i += blockDim.x) {
    const int hh = i / 128, c = i % 128;
    qc[hh][c] = p.QQ[(long long)b * p.qq_ld + heads[hh] * 128 + c];
  }
  __syncthreads();
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(p.W_UKt) + (long long)j * 128 * 512;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.qt);
  for (int l = threadIdx.x; l < 512; l += blockDim.x) {
    float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < 128; ++c) {
      const float w = __bfloat162float(W[c * 512 + l]);
#pragma unroll
      for (int hh = 0; hh < 5; ++hh) acc[hh] += w * qc[hh][c];
    }
#pragma unroll
    for (int hh = 0; hh < 5; ++hh)
      out[((long long)b * p.n_heads + heads[hh]) * 576 + l] = __float2bfloat16_rn(acc[hh]);
  }
  for (int i = threadIdx.x; i < 5 * 64; i += blockDim.x) {
    const int hh = i / 64, r = i % 64;
    out[((long long)b * p.n_heads + heads[hh]) * 576 + 512 + r] =
        __float2bfloat16_rn(p.QQ[(long long)b * p.qq_ld + p.rope_col0 + heads[hh] * 64 + r]);
  }
}

int launch_qtilde(const DecQParams& p, cudaStream_t st) {
  dim3 grid(p.B, p.n_groups);
  qtilde_kernel<<<grid, 256, 0, st>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// ---------------------------------------------------------------- split-K latent attention
// CUDA-core reference kernel: CTA (split, b) walks 64-position chunks of its key range.
namespace dec {
constexpr int CH = 64;            // positions per chunk
constexpr int RW = 289;           // padded row stride in 32-bit words (576 bf16 = 288 words)
constexpr int NH = 80;
constexpr int SMEM = (NH * RW + CH * RW) * 4 + NH * CH * 4 + NH * 4 * 3;
}  // namespace dec

__global__ void __launch_bounds__(256, 1) dec_attn_simt_kernel(DecAttnParams p) {
  using namespace dec;
  extern __shared__ uint32_t sm[];
  uint32_t* q_s = sm;                  // [80][RW] bf16x2
  uint32_t* c_s = q_s + NH * RW;       // [64][RW]
  float* sc = reinterpret_cast<float*>(c_s + CH * RW);   // [80][64]
  float* m_s = sc + NH * CH;
  float* l_s = m_s + NH;
  float* a_s = l_s + NH;
  const int sp = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  int L = p.cache_len[b];                        // keys 0..L (L cached + the new token)
  if (L < 0 || L >= p.cap) {                     // reported; the sequence reads nothing
    if (tid == 0) atomicCAS(p.err, 0, SITE_BAD_CACHE_LEN);
    L = -1;
  }
  const int lo_all = p.window > 0 ? max(0, L - p.window + 1) : 0;
  const int n_all = L - lo_all + 1;
  const int per = (n_all + p.n_split - 1) / p.n_split;
  const int lo = lo_all + sp * per;
  const int hi = min(L, lo + per - 1);
  const uint32_t* qsrc = reinterpret_cast<const uint32_t*>(p.qt) + (long long)b * NH * 288;
  for (int i = tid; i < NH * 288; i += blockDim.x) q_s[(i / 288) * RW + i % 288] = qsrc[i];
  if (tid < NH) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  float acc[NH][2];
#pragma unroll
  for (int h = 0; h < NH; ++h) acc[h][0] = acc[h][1] = 0.f;
  const uint32_t* cache = reinterpret_cast<const uint32_t*>(p.cache) + (long long)b * p.cap * 288;
  __syncthreads();
  for (int p0 = lo; p0 <= hi; p0 += CH) {
    const int np = min(CH, hi - p0 + 1);
    for (int i = tid; i < CH * 72; i += blockDim.x) {   // 72 uint4 per row
      const int r = i / 72, w4 = i % 72;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < np) v = reinterpret_cast<const uint4*>(cache + (long long)(p0 + r) * 288)[w4];
      uint32_t* d = c_s + r * RW + w4 * 4;
      d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    }
    __syncthreads();
    for (int idx = tid; idx < NH * CH; idx += blockDim.x) {
      const int h = idx / CH, r = idx % CH;
      float s = -INFINITY;
      if (r < np) {
        const uint32_t* qa = q_s + h * RW;
        const uint32_t* ca = c_s + r * RW;
        float a0 = 0.f, a1 = 0.f;
        for (int w = 0; w < 288; ++w) {
          const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(qa + w);
          const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(ca + w);
          a0 = fmaf(__low2float(x), __low2float(y), a0);
          a1 = fmaf(__high2float(x), __high2float(y), a1);
        }
        s = (a0 + a1) * p.scale_log2;
      }
      sc[h * CH + r] = s;
    }
    __syncthreads();
    if (tid < NH) {
      float mx = m_s[tid];
      for (int r = 0; r < np; ++r) mx = fmaxf(mx, sc[tid * CH + r]);
      const float alpha = ex2_approx(m_s[tid] - mx);  // m_s = -inf first: 0
      float l = l_s[tid] * alpha;
      for (int r = 0; r < CH; ++r) {
        const float e = r < np ? ex2_approx(sc[tid * CH + r] - mx) : 0.f;
        sc[tid * CH + r] = e;
        l += e;
      }
      m_s[tid] = mx;
      l_s[tid] = l;
      a_s[tid] = alpha;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      acc[h][0] *= a_s[h];
      acc[h][1] *= a_s[h];
    }
    for (int r = 0; r < np; ++r) {
      const __nv_bfloat162 cv = *reinterpret_cast<const __nv_bfloat162*>(c_s + r * RW + tid);
      const float c0 = __low2float(cv), c1 = __high2float(cv);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float pr = sc[h * CH + r];
        acc[h][0] = fmaf(pr, c0, acc[h][0]);
        acc[h][1] = fmaf(pr, c1, acc[h][1]);
      }
    }
    __syncthreads();
  }
  // partial results: latent accumulator (relative to m), and (m, l) per head
  float* part = p.part + ((long long)b * p.n_split + sp) * NH * 512;
#pragma unroll
  for (int h = 0; h < NH; ++h)
    *reinterpret_cast<float2*>(part + h * 512 + 2 * tid) = make_float2(acc[h][0], acc[h][1]);
  if (tid < NH) {
    float* ml = p.ml + (((long long)b * p.n_split + sp) * NH + tid) * 2;
    ml[0] = m_s[tid];
    ml[1] = l_s[tid];
  }
}

int launch_dec_attn_simt(const DecAttnParams& p, cudaStream_t st) {
  if (cudaFuncSetAttribute(dec_attn_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           dec::SMEM) != cudaSuccess)
    return -4;
  dim3 grid(p.n_split, p.B);
  dec_attn_simt_kernel<<<grid, 256, dec::SMEM, st>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// ---------------------------------------------------------------- split merge + combine + gate
// CTA (b, j): merges the splits of the group's 5 heads, forms the latent differential
// l_s - lambda_s l_noise for its 4 signal heads, up-projects with W_UV_j and applies the gate.
__global__ void __launch_bounds__(256) dec_combine_kernel(DecCombParams p) {
  const int b = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  constexpr int NH = 80;
  __shared__ float lat[5][512];
  __shared__ float wsp[64][5];
  __shared__ float inv_L[5];
  const int heads[5] = {p.n_signal + j, 4 * j, 4 * j + 1, 4 * j + 2, 4 * j + 3};
  if (tid < 5) {
    const int h = heads[tid];
    float M = -INFINITY;
    for (int sp = 0; sp < p.n_split; ++sp)
      M = fmaxf(M, p.ml[(((long long)b * p.n_split + sp) * NH + h) * 2]);
    float Ls = 0.f;
    for (int sp = 0; sp < p.n_split; ++sp) {
      const float* ml = p.ml + (((long long)b * p.n_split + sp) * NH + h) * 2;
      const float w = ml[1] > 0.f ? ex2_approx(ml[0] - M) : 0.f;
      wsp[sp][tid] = w;
      Ls += w * ml[1];
    }
    inv_L[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
  __syncthreads();
  for (int i = tid; i < 5 * 512; i += blockDim.x) {
    const int hh = i / 512, l = i % 512;
    float a = 0.f;
    for (int sp = 0; sp < p.n_split; ++sp)
      a += wsp[sp][hh] * p.part[(((long long)b * p.n_split + sp) * NH + heads[hh]) * 512 + l];
    lat[hh][l] = a * inv_L[hh];
  }
  __syncthreads();
  // latent differential, in place for the 4 signal heads
  for (int i = tid; i < 4 * 512; i += blockDim.x) {
    const int s = i / 512, l = i % 512;
    const float lam = p.lam[(long long)b * p.n_signal + 4 * j + s];
    lat[1 + s][l] -= lam * lat[0][l];
  }
  __syncthreads();
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(p.W_bKV);
  const int ldw = p.n_groups * 256;
  for (int o = tid; o < 4 * 128; o += blockDim.x) {
    const int s = o / 128, c = o % 128;
    float d = 0.f;
    for (int l = 0; l < 512; ++l)
      d = fmaf(lat[1 + s][l], __bfloat162float(W[(long long)l * ldw + j * 256 + 128 + c]), d);
    const int sig = 4 * j + s;
    const float g = __bfloat162float(static_cast<const __nv_bfloat16*>(p.G)[(long long)b * p.n_signal * 128 + sig * 128 + c]);
    static_cast<__nv_bfloat16*>(p.Dg)[(long long)b * p.n_signal * 128 + sig * 128 + c] =
        __float2bfloat16_rn(sigmoidf_fast(g) * d);
  }
}

int launch_dec_combine(const DecCombParams& p, cudaStream_t st) {
  dim3 grid(p.B, p.n_groups);
  dec_combine_kernel<<<grid, 256, 0, st>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
