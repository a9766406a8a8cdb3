// Down-projection epilogue of GDLA: one warp per token.
//
// From the fp32 row [x W_a^Q | x W_a^KV | x W^lambda] it forms (picx.dev "Motif 3" summary,
// section 2.2; paperglide.net Figure 1 caption):
//   c^Q      = RMSNorm(x W_a^Q)                          -> bf16 (operand of the up-projections)
//   c_bar^KV = RMSNorm(c^KV)                             -> bf16 latent-cache row, columns 0..kv_rank-1
//   k^R      = RoPE(k^R, pos) (not normalised)           -> bf16 latent-cache row, last d_rope columns
//                                                           (+ an fp16 copy for the prefill attention)
//   lambda   = sigmoid(x W^lambda), one per signal head  -> fp32
// Position: prefill row m is token m % T of sequence m / T; decode row b is at pos_ptr[b].
#include "gdla_common.cuh"
#include "gdla_fp8.cuh"
#include "gdla_internal.h"

namespace gdla {


template <int NQ, int NKV>  // per-lane element counts: q_rank / 32, kv_rank / 32
__global__ void __launch_bounds__(256) norm_rope_kernel(const __grid_constant__ NormParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= p.M) return;
  const int m = warp;
  const float* row = p.D1 + (long long)m * p.ld1;
  const __nv_bfloat16* g_q = static_cast<const __nv_bfloat16*>(p.g_q);
  const __nv_bfloat16* g_kv = static_cast<const __nv_bfloat16*>(p.g_kv);
  __nv_bfloat16* cQ = static_cast<__nv_bfloat16*>(p.cQ);
  __nv_bfloat16* latent = static_cast<__nv_bfloat16*>(p.latent);
  __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(p.cache);
  __half* kR16 = static_cast<__half*>(p.kR16);
  const int row_w = p.kv_rank + 64;

  // ---- c^Q: lane owns float4 groups lane, lane + 32, ...
  float q[NQ];
#pragma unroll
  for (int k = 0; k < NQ / 4; ++k) {
    const float4 v = *reinterpret_cast<const float4*>(row + 4 * (lane + 32 * k));
    q[4 * k] = v.x; q[4 * k + 1] = v.y; q[4 * k + 2] = v.z; q[4 * k + 3] = v.w;
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NQ; ++i) ss += q[i] * q[i];
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rq = rsqrtf(ss / float(p.q_rank) + p.eps);
#pragma unroll
  for (int k = 0; k < NQ / 4; ++k) {
    const int c = 4 * (lane + 32 * k);
    float g[4] = {1.f, 1.f, 1.f, 1.f};
    if (g_q) {
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = __bfloat162float(g_q[c + e]);
    }
    uint2 pk;
    pk.x = pack_bf162(q[4 * k] * rq * g[0], q[4 * k + 1] * rq * g[1]);
    pk.y = pack_bf162(q[4 * k + 2] * rq * g[2], q[4 * k + 3] * rq * g[3]);
    *reinterpret_cast<uint2*>(cQ + (long long)m * p.q_rank + c) = pk;
  }

  // ---- c^KV
  const float* rkv = row + p.q_rank;
  float kv[NKV];
#pragma unroll
  for (int k = 0; k < NKV / 4; ++k) {
    const float4 v = *reinterpret_cast<const float4*>(rkv + 4 * (lane + 32 * k));
    kv[4 * k] = v.x; kv[4 * k + 1] = v.y; kv[4 * k + 2] = v.z; kv[4 * k + 3] = v.w;
  }
  ss = 0.f;
#pragma unroll
  for (int i = 0; i < NKV; ++i) ss += kv[i] * kv[i];
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rkvn = rsqrtf(ss / float(p.kv_rank) + p.eps);

  // ---- k^R rotation: lane owns the pair (lane, lane + 32)
  const int qps = p.q_per_seq > 1 ? p.q_per_seq : 1;
  int pos = (p.pos_ptr ? p.pos_ptr[m / qps] + m % qps : ((m + p.row_off) % p.pos_T)) + p.pos_off;
  const int seq = p.pos_ptr ? m / qps : ((m + p.row_off) / p.pos_T);
  bool cache_ok = p.cache != nullptr;
  if (cache_ok && (pos < 0 || pos >= p.cache_cap)) {
    if (lane == 0 && p.err) atomicCAS(p.err, 0, SITE_BAD_CACHE_LEN);
    cache_ok = false;
    pos = 0;
  }
  const float* rkr = rkv + p.kv_rank;
  float cs, sn;
  rope_cs(pos, p.rope.inv_freq[lane], &cs, &sn);
  const float x1 = rkr[lane], x2 = rkr[lane + 32];
  const float k1 = x1 * cs - x2 * sn, k2 = x2 * cs + x1 * sn;

  __nv_bfloat16* dsts[2] = {latent ? latent + (long long)m * row_w : nullptr,
                            cache_ok ? cache + ((long long)seq * p.cache_cap + pos) * row_w : nullptr};
#pragma unroll
  for (int d = 0; d < 2; ++d) {
    __nv_bfloat16* dst = dsts[d];
    if (!dst) continue;
#pragma unroll
    for (int k = 0; k < NKV / 4; ++k) {
      const int c = 4 * (lane + 32 * k);
      float g[4] = {1.f, 1.f, 1.f, 1.f};
      if (g_kv) {
#pragma unroll
        for (int e = 0; e < 4; ++e) g[e] = __bfloat162float(g_kv[c + e]);
      }
      uint2 pk;
      pk.x = pack_bf162(kv[4 * k] * rkvn * g[0], kv[4 * k + 1] * rkvn * g[1]);
      pk.y = pack_bf162(kv[4 * k + 2] * rkvn * g[2], kv[4 * k + 3] * rkvn * g[3]);
      *reinterpret_cast<uint2*>(dst + c) = pk;
    }
    dst[p.kv_rank + lane] = __float2bfloat16_rn(k1);
    dst[p.kv_rank + lane + 32] = __float2bfloat16_rn(k2);
  }
  if (kR16) {
    bool bad = false;
    kR16[(long long)m * 64 + lane] = half_sat(k1, bad);
    kR16[(long long)m * 64 + lane + 32] = half_sat(k2, bad);
    if (bad && p.err) atomicCAS(p.err, 0, SITE_FP16_RANGE);
  }

  // ---- lambda
  const float* rl = rkr + 64;
  for (int c = lane; c < p.n_signal; c += 32)
    p.lam[(long long)m * p.n_signal + c] = 1.0f / (1.0f + expf(-rl[c]));
}

// The same epilogue with one CTA of 256 threads per token (q_rank 1024, kv_rank 512): for the
// few rows of a decode step, where one warp per token would leave the step waiting on a single
// warp's chain of loads, reductions and stores.  Thread t owns c^Q columns 4t .. 4t + 3 and,
// for t < 128, c^KV columns 4t .. 4t + 3; warp 0 rotates k^R (pair lane, lane + 32); threads
// t < n_signal form lambda.
__global__ void __launch_bounds__(256) norm_rope_row_kernel(const __grid_constant__ NormParams p) {
  __shared__ float red[2][8];
  const int m = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const float* row = p.D1 + (long long)m * p.ld1;
  const __nv_bfloat16* g_q = static_cast<const __nv_bfloat16*>(p.g_q);
  const __nv_bfloat16* g_kv = static_cast<const __nv_bfloat16*>(p.g_kv);
  const int row_w = p.kv_rank + 64;
  const float4 q4 = *reinterpret_cast<const float4*>(row + 4 * t);
  const bool has_kv = t < 128;
  const float4 kv4 = has_kv ? *reinterpret_cast<const float4*>(row + p.q_rank + 4 * t) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float* rkr = row + p.q_rank + p.kv_rank;
  const float x1 = warp == 0 ? rkr[lane] : 0.f, x2 = warp == 0 ? rkr[lane + 32] : 0.f;
  const float xl = t < p.n_signal ? rkr[64 + t] : 0.f;
  float sq = q4.x * q4.x + q4.y * q4.y + q4.z * q4.z + q4.w * q4.w;
  float sk = kv4.x * kv4.x + kv4.y * kv4.y + kv4.z * kv4.z + kv4.w * kv4.w;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    sk += __shfl_xor_sync(0xffffffffu, sk, o);
  }
  if (lane == 0) {
    red[0][warp] = sq;
    red[1][warp] = sk;
  }
  __syncthreads();
  float tq = 0.f, tk = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    tq += red[0][w];
    tk += red[1][w];
  }
  const float rq = rsqrtf(tq / float(p.q_rank) + p.eps);
  const float rkvn = rsqrtf(tk / float(p.kv_rank) + p.eps);
  {
    float g[4] = {1.f, 1.f, 1.f, 1.f};
    if (g_q) {
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = __bfloat162float(g_q[4 * t + e]);
    }
    uint2 pk;
    pk.x = pack_bf162(q4.x * rq * g[0], q4.y * rq * g[1]);
    pk.y = pack_bf162(q4.z * rq * g[2], q4.w * rq * g[3]);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.cQ) + (long long)m * p.q_rank + 4 * t) = pk;
  }
  const int qps = p.q_per_seq > 1 ? p.q_per_seq : 1;
  int pos = (p.pos_ptr ? p.pos_ptr[m / qps] + m % qps : ((m + p.row_off) % p.pos_T)) + p.pos_off;
  const int seq = p.pos_ptr ? m / qps : ((m + p.row_off) / p.pos_T);
  bool cache_ok = p.cache != nullptr;
  if (cache_ok && (pos < 0 || pos >= p.cache_cap)) {
    if (t == 0 && p.err) atomicCAS(p.err, 0, SITE_BAD_CACHE_LEN);
    cache_ok = false;
    pos = 0;
  }
  const bool c8 = p.cache_fp8 != 0;
  __nv_bfloat16* dsts[2] = {p.latent ? static_cast<__nv_bfloat16*>(p.latent) + (long long)m * row_w : nullptr,
                            cache_ok && !c8 ? static_cast<__nv_bfloat16*>(p.cache) + ((long long)seq * p.cache_cap + pos) * row_w
                                            : nullptr};
  // MXFP8 cache row (gdla_fp8.cuh): the bf16-rounded values, 32 per block (8 threads here)
  uint8_t* row8 = cache_ok && c8 ? static_cast<uint8_t*>(p.cache) + ((long long)seq * p.cache_cap + pos) * FP8_ROW_BYTES
                                 : nullptr;
  if (row8 && t < 128) {
    float g[4] = {1.f, 1.f, 1.f, 1.f};
    if (g_kv) {
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = __bfloat162float(g_kv[4 * t + e]);
    }
    const float b0 = __bfloat162float(__float2bfloat16_rn(kv4.x * rkvn * g[0]));
    const float b1 = __bfloat162float(__float2bfloat16_rn(kv4.y * rkvn * g[1]));
    const float b2 = __bfloat162float(__float2bfloat16_rn(kv4.z * rkvn * g[2]));
    const float b3 = __bfloat162float(__float2bfloat16_rn(kv4.w * rkvn * g[3]));
    float amax = fmaxf(fmaxf(fabsf(b0), fabsf(b1)), fmaxf(fabsf(b2), fabsf(b3)));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int k = mx_block_exp(amax);
    const float inv = exp2i(-k);
    *reinterpret_cast<uint32_t*>(row8 + 4 * t) =
        uint32_t(e4m3x2_from(b0 * inv, b1 * inv)) | (uint32_t(e4m3x2_from(b2 * inv, b3 * inv)) << 16);
    if ((t & 7) == 0) row8[FP8_SCALE_OFF + (t >> 3)] = uint8_t(k + 127);
  }
  if (has_kv) {
    float g[4] = {1.f, 1.f, 1.f, 1.f};
    if (g_kv) {
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = __bfloat162float(g_kv[4 * t + e]);
    }
    uint2 pk;
    pk.x = pack_bf162(kv4.x * rkvn * g[0], kv4.y * rkvn * g[1]);
    pk.y = pack_bf162(kv4.z * rkvn * g[2], kv4.w * rkvn * g[3]);
#pragma unroll
    for (int d = 0; d < 2; ++d)
      if (dsts[d]) *reinterpret_cast<uint2*>(dsts[d] + 4 * t) = pk;
  }
  if (warp == 0) {
    float cs, sn;
    rope_cs(pos, p.rope.inv_freq[lane], &cs, &sn);
    const float k1 = x1 * cs - x2 * sn, k2 = x2 * cs + x1 * sn;
#pragma unroll
    for (int d = 0; d < 2; ++d) {
      if (!dsts[d]) continue;
      dsts[d][p.kv_rank + lane] = __float2bfloat16_rn(k1);
      dsts[d][p.kv_rank + lane + 32] = __float2bfloat16_rn(k2);
    }
    if (row8) {
      // rope dims 0..31 form block 16 and 32..63 block 17 (one value per lane each)
      const float r1 = __bfloat162float(__float2bfloat16_rn(k1)), r2 = __bfloat162float(__float2bfloat16_rn(k2));
      float a1 = fabsf(r1), a2 = fabsf(r2);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, o));
        a2 = fmaxf(a2, __shfl_xor_sync(0xffffffffu, a2, o));
      }
      const int k16 = mx_block_exp(a1), k17 = mx_block_exp(a2);
      row8[p.kv_rank + lane] = uint8_t(e4m3x2_from(r1 * exp2i(-k16), 0.f) & 0xFFu);
      row8[p.kv_rank + 32 + lane] = uint8_t(e4m3x2_from(r2 * exp2i(-k17), 0.f) & 0xFFu);
      if (lane == 0) {
        row8[FP8_SCALE_OFF + 16] = uint8_t(k16 + 127);
        row8[FP8_SCALE_OFF + 17] = uint8_t(k17 + 127);
      }
      if (lane >= 1 && lane <= FP8_ROW_BYTES - FP8_SCALE_OFF - 18) row8[FP8_SCALE_OFF + 17 + lane] = 0;
    }
    if (p.kR16) {
      __half* kR16 = static_cast<__half*>(p.kR16);
      bool bad = false;
      kR16[(long long)m * 64 + lane] = half_sat(k1, bad);
      kR16[(long long)m * 64 + lane + 32] = half_sat(k2, bad);
      if (bad && p.err) atomicCAS(p.err, 0, SITE_FP16_RANGE);
    }
  }
  if (t < p.n_signal) p.lam[(long long)m * p.n_signal + t] = 1.0f / (1.0f + expf(-xl));
}

// fp16 copy of the rotated k^R of bf16 latent rows (a key prefix handed in by the caller)
__global__ void latent_to_kr16_kernel(const __nv_bfloat16* __restrict__ latent, int row_w,
                                      int kv_rank, long long rows, __half* __restrict__ kR16, int* err) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * 64) return;
  const long long m = i >> 6;
  bool bad = false;
  kR16[i] = half_sat(__bfloat162float(latent[m * row_w + kv_rank + (i & 63)]), bad);
  if (bad && err) atomicCAS(err, 0, SITE_FP16_RANGE);
}

int launch_latent_to_kr16(const void* latent, int kv_rank, long long rows, void* kR16, int* err,
                          cudaStream_t st) {
  if (rows <= 0) return 0;
  const long long n = rows * 64;
  latent_to_kr16_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(latent), kv_rank + 64, kv_rank, rows, static_cast<__half*>(kR16), err);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

int launch_norm_rope(const NormParams& p, cudaStream_t st) {
  if (p.M <= 0) return 0;
  const int threads = 256;
  const int blocks = (p.M * 32 + threads - 1) / threads;
  if (p.q_rank == 1024 && p.kv_rank == 512 && (p.M <= 4096 || p.cache_fp8) && p.n_signal <= 256)
    norm_rope_row_kernel<<<p.M, 256, 0, st>>>(p);      // few rows (or an MXFP8 cache): a CTA per token
  else if (p.cache_fp8)
    return -2;
  else if (p.q_rank == 1024 && p.kv_rank == 512)
    norm_rope_kernel<32, 16><<<blocks, threads, 0, st>>>(p);
  else if (p.q_rank == 128 && p.kv_rank == 128)
    norm_rope_kernel<4, 4><<<blocks, threads, 0, st>>>(p);
  else
    return -2;
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
