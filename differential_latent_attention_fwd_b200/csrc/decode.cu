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
// Kernels here: W_UK transpose (weight absorption), q~ formation, and the split merge +
// latent differential combine + W_UV up-projection + gate.  The split-K latent attention
// itself is the tensor-core kernel in decode_tc.cu.
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
// CTA (KV head j, 4 rows b): W_UK_j^T (128 x 512 bf16, 128 KB) is staged in shared memory with
// asynchronous copies, then 20 query rows (4 rows x the group's 5 heads) are projected.
__global__ void __launch_bounds__(256) qtilde_kernel(DecQParams p) {
  extern __shared__ uint8_t qt_smem[];
  __nv_bfloat16* wsm = reinterpret_cast<__nv_bfloat16*>(qt_smem);            // [128][512]
  float (*qc)[128] = reinterpret_cast<float (*)[128]>(qt_smem + 128 * 512 * 2);  // [20][128]
  const int j = blockIdx.x, b0 = blockIdx.y * 4, tid = threadIdx.x;
  const int nb = min(4, p.B - b0);
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(p.W_UKt) + (long long)j * 128 * 512;
  for (int i = tid; i < 128 * 512 / 8; i += blockDim.x) cp_async16(wsm + i * 8, W + i * 8);
  const int heads[5] = {p.n_signal + j, 4 * j, 4 * j + 1, 4 * j + 2, 4 * j + 3};
  for (int i = tid; i < 20 * 128; i += blockDim.x) {
    const int r = i / 128, c = i % 128, bb = r / 5, hh = r % 5;
    qc[r][c] = bb < nb ? p.QQ[(long long)(b0 + bb) * p.qq_ld + heads[hh] * 128 + c] : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  // thread: latent columns 2 tid, 2 tid + 1 of all 20 rows
  float acc[20][2];
#pragma unroll
  for (int r = 0; r < 20; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll 2
  for (int c = 0; c < 128; ++c) {
    const __nv_bfloat162 w2 = *reinterpret_cast<const __nv_bfloat162*>(wsm + c * 512 + 2 * tid);
    const float w0 = __low2float(w2), w1 = __high2float(w2);
#pragma unroll
    for (int r = 0; r < 20; ++r) {
      const float q = qc[r][c];
      acc[r][0] = fmaf(q, w0, acc[r][0]);
      acc[r][1] = fmaf(q, w1, acc[r][1]);
    }
  }
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.qt);
#pragma unroll
  for (int r = 0; r < 20; ++r) {
    const int bb = r / 5, hh = r % 5;
    if (bb >= nb) continue;
    *reinterpret_cast<uint32_t*>(out + ((long long)(b0 + bb) * p.n_heads + heads[hh]) * 576 + 2 * tid) =
        pack_bf162(acc[r][0], acc[r][1]);
  }
  for (int i = tid; i < 4 * 5 * 64; i += blockDim.x) {
    const int r = i / 64, e = i % 64, bb = r / 5, hh = r % 5;
    if (bb >= nb) continue;
    out[((long long)(b0 + bb) * p.n_heads + heads[hh]) * 576 + 512 + e] =
        __float2bfloat16_rn(p.QQ[(long long)(b0 + bb) * p.qq_ld + p.rope_col0 + heads[hh] * 64 + e]);
  }
}

int launch_qtilde(const DecQParams& p, cudaStream_t st) {
  const int smem = 128 * 512 * 2 + 20 * 128 * 4;
  if (cudaFuncSetAttribute(qtilde_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return -4;
  qtilde_kernel<<<dim3(p.n_groups, (p.B + 3) / 4), 256, smem, st>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// ---------------------------------------------------------------- split merge + combine + gate
// Kernel 1, CTA (b, j): merges the splits of the group's 5 heads (rescaling each split's
// partial by 2^(m_split - m)), normalises, and forms the latent differential
// l_s - lambda_s l_noise for the group's 4 signal heads -> Dlat[j][b * 4 + s][512] (fp32).
__global__ void __launch_bounds__(256) dec_merge_kernel(DecCombParams p) {
  const int b = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;
  constexpr int NH = 80;
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
  for (int l = tid; l < 512; l += blockDim.x) {
    float lat[5];
#pragma unroll
    for (int hh = 0; hh < 5; ++hh) {
      float a = 0.f;
      for (int sp = 0; sp < p.n_split; ++sp) {
        const float w = wsp[sp][hh];
        if (w != 0.f)  // empty splits write no partial
          a += w * p.part[(((long long)b * p.n_split + sp) * NH + heads[hh]) * 512 + l];
      }
      lat[hh] = a * inv_L[hh];
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const float lam = p.lam[(long long)b * p.n_signal + 4 * j + s];
      p.Dlat[((long long)j * p.B + b) * 4 * 512 + s * 512 + l] = lat[1 + s] - lam * lat[0];
    }
  }
}

// Kernel 2, CTA (j, 4 sequences): D = Dlat W_UV_j (16 rows x 128 columns, K = 512), then
// Dg = sigmoid(G) (.) D.  W_UV_j is the V column block of W_b^KV for KV head j; it is staged
// in shared memory (128 KB, coalesced 16-byte loads) before the product.
__global__ void __launch_bounds__(256) dec_uv_gate_kernel(DecCombParams p) {
  extern __shared__ uint8_t uv_smem[];
  float (*dl)[512] = reinterpret_cast<float (*)[512]>(uv_smem);                      // [16][512]
  __nv_bfloat16* wsm = reinterpret_cast<__nv_bfloat16*>(uv_smem + 16 * 512 * 4);     // [512][128]
  const int j = blockIdx.x, b0 = blockIdx.y * 4, tid = threadIdx.x;
  const int nrows = min(4, p.B - b0) * 4;
  const long long ldw = (long long)p.n_groups * 256;
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(p.W_bKV) + j * 256 + 128;
  for (int i = tid; i < 512 * 16; i += blockDim.x) {          // 16 x 16 bytes per 128-column row
    const int l = i >> 4, q = i & 15;
    cp_async16(wsm + l * 128 + q * 8, W + l * ldw + q * 8);
  }
  const float* src = p.Dlat + ((long long)j * p.B + b0) * 4 * 512;
  for (int i = tid; i < 16 * 512; i += blockDim.x)
    dl[i / 512][i % 512] = (i / 512) < nrows ? src[i] : 0.f;
  cp_async_wait_all();
  __syncthreads();
  const int cq = tid & 31;          // columns 4 cq .. 4 cq + 3
  const int rp = tid >> 5;          // rows 2 rp, 2 rp + 1
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
  for (int l = 0; l < 512; ++l) {
    const uint2 wv = *reinterpret_cast<const uint2*>(wsm + l * 128 + 4 * cq);
    const __nv_bfloat162 w01 = *reinterpret_cast<const __nv_bfloat162*>(&wv.x);
    const __nv_bfloat162 w23 = *reinterpret_cast<const __nv_bfloat162*>(&wv.y);
    const float w[4] = {__low2float(w01), __high2float(w01), __low2float(w23), __high2float(w23)};
    const float d0 = dl[2 * rp][l], d1 = dl[2 * rp + 1][l];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[0][e] = fmaf(d0, w[e], acc[0][e]);
      acc[1][e] = fmaf(d1, w[e], acc[1][e]);
    }
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = 2 * rp + rr;
    if (row >= nrows) continue;
    const int b = b0 + row / 4, s = row % 4, sig = 4 * j + s;
    const long long o = (long long)b * p.n_signal * 128 + sig * 128 + 4 * cq;
    const uint2 gv = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p.G) + o);
    const __nv_bfloat162 g01 = *reinterpret_cast<const __nv_bfloat162*>(&gv.x);
    const __nv_bfloat162 g23 = *reinterpret_cast<const __nv_bfloat162*>(&gv.y);
    uint2 out;
    out.x = pack_bf162(sigmoidf_fast(__low2float(g01)) * acc[rr][0], sigmoidf_fast(__high2float(g01)) * acc[rr][1]);
    out.y = pack_bf162(sigmoidf_fast(__low2float(g23)) * acc[rr][2], sigmoidf_fast(__high2float(g23)) * acc[rr][3]);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.Dg) + o) = out;
  }
}

int launch_dec_combine(const DecCombParams& p, cudaStream_t st) {
  dec_merge_kernel<<<dim3(p.B, p.n_groups), 256, 0, st>>>(p);
  if (cudaPeekAtLastError() != cudaSuccess) return -4;
  const int uv_smem = 16 * 512 * 4 + 512 * 128 * 2;
  if (cudaFuncSetAttribute(dec_uv_gate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, uv_smem) !=
      cudaSuccess)
    return -4;
  dec_uv_gate_kernel<<<dim3(p.n_groups, (p.B + 3) / 4), 256, uv_smem, st>>>(p);
  if (cudaPeekAtLastError() != cudaSuccess) return -4;
  count_extra_launch();
  return 0;
}

}  // namespace gdla
