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
// Kernels here: W_UK transpose (weight absorption), q~ formation, and the segment merge +
// latent differential combine + W_UV up-projection + gate (one kernel).  The latent attention
// itself (one wave of CTAs over the key tiles of all rows) is the tensor-core kernel in
// decode_tc.cu.
#include "gdla_common.cuh"
#include "gdla_internal.h"
#include "gdla_decode.h"

namespace gdla {

// W_UKt[j][c][l] = W_bKV[l][j * (d_nope + d_v) + c], in fp16 (the operand type of the q~ MMAs;
// exact for weights of magnitude >= 2^-14, the fp16 normal range)
__global__ void absorb_uk_kernel(const __nv_bfloat16* __restrict__ W_bKV, __half* __restrict__ W_UKt,
                                 int kv_rank, int n_kv, int d_nope, int d_v) {
  const long long total = (long long)n_kv * d_nope * kv_rank;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int l = int(i % kv_rank);
    const int c = int((i / kv_rank) % d_nope);
    const int j = int(i / ((long long)kv_rank * d_nope));
    W_UKt[i] = __float2half_rn(__bfloat162float(W_bKV[(long long)l * n_kv * (d_nope + d_v) + j * (d_nope + d_v) + c]));
  }
}

int launch_absorb_uk(const void* W_bKV, void* W_UKt, int kv_rank, int n_kv, int d_nope, int d_v,
                     cudaStream_t st) {
  absorb_uk_kernel<<<1024, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W_bKV),
                                         static_cast<__half*>(W_UKt), kv_rank, n_kv, d_nope, d_v);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

__global__ void copy_cols_kernel(const uint4* __restrict__ src, long long ld_src8, uint4* __restrict__ dst,
                                 long long ld_dst8, long long col0_8, int rows, int cols8) {
  const long long total = (long long)rows * cols8;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols8, c = i % cols8;
    dst[r * ld_dst8 + col0_8 + c] = src[r * ld_src8 + c];
  }
}

int launch_copy_cols(const void* src, long long ld_src, void* dst, long long ld_dst, int col0, int rows,
                     int cols, cudaStream_t st) {
  if ((cols | col0) % 8 || ld_src % 8 || ld_dst % 8) return -1;
  copy_cols_kernel<<<1024, 256, 0, st>>>(static_cast<const uint4*>(src), ld_src / 8, static_cast<uint4*>(dst),
                                         ld_dst / 8, col0 / 8, rows, cols / 8);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// q~ rows: qt[b][h][0..511] = W_UK_j q^C_h, qt[b][h][512..575] = rotated q^R_h (bf16), on the
// tensor cores.  Per KV head j the rows (b, h) of its five heads form one product
//   [5 B x 128] (q^C, fp16) x [128 x 512] (W_UK_j^T, fp16) -> fp32 in TMEM,
// one CTA per (j, 128 rows, 128 of the 512 columns), so that a decode batch fills the SMs (three
// CTAs fit on one): the q^C rows are converted to fp16 by the CTA's threads into a
// 128-byte-swizzled K-major tile, the CTA's quarter of W_UK_j^T (32 KB) arrives by TMA as two
// [128][64] MN-major boxes, and one tcgen05.mma chain (M 128, N 128, K 128) fills 128 TMEM
// columns; while it runs the CTA copies its share of the rotated q^R rows.  The four warps
// (thread = row) round the result to bf16 into shared memory, from where whole 256-byte row
// pieces go out coalesced.  Rows of the group: r = 5 b + hh, hh = 0 the noise head n_signal + j,
// hh = 1..4 the signal heads 4 j + hh - 1.
namespace qtc {
constexpr int NQ = 4;                         // column quarters of q~ (one CTA each)
constexpr int A_BOX = 128 * 128;              // [128 rows][64 fp16]
constexpr int B_BOX = 128 * 128;              // [128 K rows][64 N fp16]
constexpr int A_OFF = 0, B_OFF = 2 * A_BOX;
constexpr int BAR_OFF = B_OFF + 2 * B_BOX;
constexpr int SMEM = BAR_OFF + 64 + 1024;
}  // namespace qtc

__device__ __forceinline__ int qt_head(int hh, int j, int n_signal) {
  return hh == 0 ? n_signal + j : 4 * j + hh - 1;
}

__global__ void __launch_bounds__(128, 3)
    qtilde_tc_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ DecQParams p, KernelCtl ctl) {
  using namespace qtc;
  extern __shared__ uint8_t qt_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qt_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* bar_mma = bar_w + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_w + 2);
  const int j = blockIdx.x, nq = blockIdx.z, t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int R = 5 * p.B;
  const int tile0 = blockIdx.y * 128;           // first group row of the tile

  if (t == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapW);
    mbar_expect_tx(bar_w, 2 * B_BOX);
#pragma unroll
    for (int c = 0; c < 2; ++c) tma_load_2d(smem + B_OFF + c * B_BOX, &mapW, bar_w, 64 * (2 * nq + c), j * 128);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  // ---- A: the q^C rows of warp w (32 w .. 32 w + 31 of the tile), one row per load (lane l:
  // float4 l), as fp16 into the 128-byte-swizzled K-major tile (two lanes per 16-byte chunk)
  const int row0 = tile0 + 32 * warp;
  bool bad = false;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float4 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int rr = row0 + 16 * half + i;
      v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rr < R)
        v[i] = *reinterpret_cast<const float4*>(p.QQ + (long long)(rr / 5) * p.qq_ld +
                                                (long long)qt_head(rr % 5, j, p.n_signal) * 128 + 4 * lane);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 32 * warp + 16 * half + i;        // row within the tile
      const int k8 = lane >> 1;                        // 8-value chunk of the 128 columns
      *reinterpret_cast<uint2*>(smem + A_OFF + (k8 >> 3) * A_BOX + r * 128 + (((k8 & 7) ^ (r & 7)) << 4) +
                                8 * (lane & 1)) =
          make_uint2(pack_half2_sat(v[i].x, v[i].y, bad), pack_half2_sat(v[i].z, v[i].w, bad));
    }
  }
  if (bad && ctl.err) atomicCAS(ctl.err, 0, SITE_FP16_RANGE);
  bad = false;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true, issued = false;
  if (t == 0) {
    ok = mbar_wait(bar_w, 0, ctl, SITE_DEC_MMA);
    if (ok) {
      tc_fence_after();
      issued = true;
      constexpr uint32_t idesc = make_idesc(128, 128, 0, 0, 1);
      const uint64_t da = sdesc_sw128(smem_u32(smem + A_OFF), 16, 1024);
      const uint64_t db = sdesc_sw128(smem_u32(smem + B_OFF), B_BOX, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss(tmem, da + uint64_t((kk >> 2) * (A_BOX >> 4) + (kk & 3) * 2), db + uint64_t(kk * 128), idesc,
               kk > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
  }
  // ---- while the MMAs run: the rotated q^R of rows 32 nq .. 32 nq + 31 of the tile (bf16, or
  // fp16 for the MXFP8 decode) straight into q~ columns 512..575, 16 lanes per row
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = 128 * i + t, rr = tile0 + 32 * nq + (idx >> 4), c4 = idx & 15;
    if (rr < R) {
      const int bb = rr / 5, hr = qt_head(rr % 5, j, p.n_signal);
      const float4 a = *reinterpret_cast<const float4*>(p.QQ + (long long)bb * p.qq_ld + p.rope_col0 +
                                                        (long long)hr * 64 + 4 * c4);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.qt) + ((long long)bb * p.n_heads + hr) * 576 + 512 +
                                4 * c4) =
          p.qt_f16 ? make_uint2(pack_half2_sat(a.x, a.y, bad), pack_half2_sat(a.z, a.w, bad))
                   : make_uint2(pack_bf162(a.x, a.y), pack_bf162(a.z, a.w));
    }
  }
  ok = __syncthreads_and(ok);
  if (ok) {
    // ---- epilogue: thread t = TMEM lane t = tile row t; its 128 values are rounded into the
    // (now free) A region as one 256-byte row, 16-byte chunk k at position k ^ (t & 15)
    const bool w = __all_sync(0xffffffffu, mbar_wait(bar_mma, 0, ctl, SITE_DEC_MMA));
    tc_fence_after();
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    auto pk = [&](float a, float b) { return p.qt_f16 ? pack_half2_sat(a, b, bad) : pack_bf162(a, b); };
    if (w) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[64];
        GDLA_TMEM_LD32(tmem + 64 * c + lane_off, v);
        GDLA_TMEM_LD32(tmem + 64 * c + 32 + lane_off, (v + 32));
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 64; e += 8) {
          const int k = (64 * c + e) >> 3;
          *reinterpret_cast<uint4*>(smem + A_OFF + t * 256 + ((k ^ (t & 15)) << 4)) =
              make_uint4(pk(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                         pk(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                         pk(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                         pk(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
        }
      }
    }
    ok = __syncthreads_and(w);
    if (ok) {
      // 16 lanes per row piece: columns 128 nq .. 128 nq + 127 of q~ row (b, h)
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int idx = 128 * i + t, r = idx >> 4, k = idx & 15, gr = tile0 + r;
        if (gr < R) {
          const int b = gr / 5, h = qt_head(gr % 5, j, p.n_signal);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.qt) + ((long long)b * p.n_heads + h) * 576 +
                                    128 * nq + 8 * k) =
              *reinterpret_cast<const uint4*>(smem + A_OFF + r * 256 + ((k ^ (r & 15)) << 4));
        }
      }
    }
  }
  if (bad && ctl.err) atomicCAS(ctl.err, 0, SITE_FP16_RANGE);
  if (t == 0) {
    // before TMEM is released: the MMAs (if issued) are complete, the weight copy has landed
    if (issued) mbar_drain(bar_mma, 0, ctl.err);
    else mbar_drain(bar_w, 0, ctl.err);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

int launch_qtilde(const DecQParams& p, KernelCtlHost ctl, cudaStream_t st) {
  CUtensorMap mw;
  if (make_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.W_UKt, 512, (uint64_t)p.n_groups * 128, 512 * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  if (cudaFuncSetAttribute(qtilde_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qtc::SMEM) != cudaSuccess)
    return -4;
  KernelCtl kc{ctl.err, ctl.limit_ns};
  qtilde_tc_kernel<<<dim3(p.n_groups, (5 * p.B + 127) / 128, qtc::NQ), 128, qtc::SMEM, st>>>(mw, p, kc);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// ---------------------------------------------------------------- segment merge + combine + gate
// CTA (KV group j, CB query rows b): while W_UV_j (the V column block of W_b^KV for KV head j,
// 512 x 128 bf16) arrives by TMA, the key-range segments of the group's 5 heads are merged (each
// segment's partial rescaled by 2^(m_seg - m), then normalised) and the latent differentials
// l_s - lambda_s l_noise of its 4 signal heads formed (fp32); then D = Dlat W_UV_j on the tensor
// cores and Dg = sigmoid(G) (.) D.  The fp32 differentials enter the bf16 MMA as two bf16 parts,
// hi = bf16(x) and lo = bf16(x - hi) (rows 4 b + s and 32 + 4 b + s of the A tile), whose
// products are added in fp32, so the product keeps about 16 bits of the differential.
// Row b's segments are the attention CTAs c_lo .. c_hi whose tile ranges meet the row's tiles
// [tstart[l], tstart[l + 1]) at list position l of row b; CTA c wrote its piece to slot c + l.
constexpr int CB = 8;
constexpr int MAXSEG = DEC_MAX_CTAS;
namespace dcb {
constexpr int A_CHUNK = 64 * 128;                  // [64 rows][64 bf16], 128-byte swizzle
constexpr int A_OFF = 0;                           // 8 chunks: K = 512
constexpr int B_OFF = 8 * A_CHUNK;                 // [2 N chunks][512 K rows][64 bf16]
constexpr int B_NCHUNK = 512 * 128;
constexpr int SCR_OFF = B_OFF + 2 * B_NCHUNK;
constexpr int SMEM = SCR_OFF + 5 * CB * MAXSEG * 4 + 5 * CB * 4 + 2 * CB * 4 + 64 + 1024;
// the M = 128 MMA reads 128 rows of each 64-row A chunk: rows 64..127 are the next chunk (the
// last chunk's: the first 8 KB of W_UV), which only feed TMEM lanes the epilogue never reads
static_assert(B_OFF + A_CHUNK <= SCR_OFF, "A over-read stays in shared memory");
}  // namespace dcb

__global__ void __launch_bounds__(256, 1)
    dec_combine_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ DecCombParams p,
                       KernelCtl ctl) {
  using namespace dcb;
  constexpr int NH = 80;
  extern __shared__ uint8_t cb_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(cb_raw) + 1023) & ~uintptr_t(1023));
  float (*wsp)[MAXSEG] = reinterpret_cast<float (*)[MAXSEG]>(smem + SCR_OFF);
  float* inv_L = reinterpret_cast<float*>(smem + SCR_OFF + 5 * CB * MAXSEG * 4);
  int* seg_lo = reinterpret_cast<int*>(inv_L + 5 * CB);
  int* seg_n = seg_lo + CB;
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(seg_n + CB);
  uint64_t* bar_mma = bar_w + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_w + 2);
  const int j = blockIdx.x, b0 = blockIdx.y * CB, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = min(CB, p.B - b0);
  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapW);
    // W_UV_j = columns j 256 + 128 .. j 256 + 255 of W_b^KV: N chunk c, K half kh
    mbar_expect_tx(bar_w, 2 * B_NCHUNK);
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int kh = 0; kh < 2; ++kh)
        tma_load_2d(smem + B_OFF + c * B_NCHUNK + kh * (B_NCHUNK / 2), &mapW, bar_w, j * 256 + 128 + 64 * c, 256 * kh);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  // the lambdas of this thread's rows, loaded now and used after the merge
  constexpr int RB = CB / 2;
  const int cq = tid & 127, rb = (tid >> 7) * RB;
  float lamv[RB][4];
#pragma unroll
  for (int k = 0; k < RB; ++k)
#pragma unroll
    for (int s = 0; s < 4; ++s)
      lamv[k][s] = rb + k < nb ? p.lam[(long long)(b0 + rb + k) * p.n_signal + 4 * j + s] : 0.f;
  if (tid < CB) {
    int lo = 0, n = 0;
    if (tid < nb) {
      const int b = b0 + tid, l = dec_list_pos(b, p.q_len, p.n_seq);
      const long long N = p.tstart[p.B], G = dec_ctas_used(N, p.n_ctas, p.q_len);
      const long long t0 = p.tstart[l], t1 = p.tstart[l + 1];
      if (t1 > t0) {
        // CTA c < G = min(grid, N) covers tiles [c N / G, (c + 1) N / G) (never empty): tile t
        // lies in CTA ((t + 1) G - 1) / N
        const int c_lo = int(((t0 + 1) * G - 1) / N), c_hi = int((t1 * G - 1) / N);
        lo = c_lo + l;
        n = c_hi - c_lo + 1;
      }
    }
    seg_lo[tid] = lo;
    seg_n[tid] = n;
  }
  __syncthreads();
  const int heads[5] = {p.n_signal + j, 4 * j, 4 * j + 1, 4 * j + 2, 4 * j + 3};
  if (tid < 5 * CB) {
    const int bb = tid / 5, h = heads[tid % 5];
    const int n = seg_n[bb], lo = seg_lo[bb];
    // (m, l) of the segments, four loads in flight at a time
    float M = -INFINITY, Ls = 0.f;
    for (int k0 = 0; k0 < n; k0 += 4) {
      float2 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = k0 + k < n ? *reinterpret_cast<const float2*>(p.ml + ((long long)(lo + k0 + k) * NH + h) * 2)
                          : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) M = fmaxf(M, v[k].x);
    }
    for (int k0 = 0; k0 < n; k0 += 4) {
      float2 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = k0 + k < n ? *reinterpret_cast<const float2*>(p.ml + ((long long)(lo + k0 + k) * NH + h) * 2)
                          : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float w = v[k].y > 0.f ? ex2_approx(v[k].x - M) : 0.f;
        if (k0 + k < n) wsp[tid][k0 + k] = w;
        Ls += w * v[k].y;
      }
    }
    inv_L[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
  __syncthreads();
  {
    // thread: latent columns 4 cq .. 4 cq + 3 of rows rb .. rb + CB / 2 - 1; segments outermost
    // so that a segment's 5 CB / 2 float4 loads are independent (rows with fewer segments load
    // nothing for the rest)
    int max_n = 0;
#pragma unroll
    for (int k = 0; k < RB; ++k) max_n = max(max_n, seg_n[rb + k]);
    float4 m4[RB][5];
#pragma unroll
    for (int k = 0; k < RB; ++k)
#pragma unroll
      for (int hh = 0; hh < 5; ++hh) m4[k][hh] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sg = 0; sg < max_n; ++sg) {
      float4 v4[RB][5];
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        const int bb = rb + k;
        const bool has = sg < seg_n[bb];
        const float* src = p.part + (long long)(has ? seg_lo[bb] + sg : 0) * NH * 512 + 4 * cq;
#pragma unroll
        for (int hh = 0; hh < 5; ++hh)
          v4[k][hh] = has ? *reinterpret_cast<const float4*>(src + (long long)heads[hh] * 512)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int k = 0; k < RB; ++k)
#pragma unroll
        for (int hh = 0; hh < 5; ++hh) {
          const float w = sg < seg_n[rb + k] ? wsp[5 * (rb + k) + hh][sg] : 0.f;
          if (w != 0.f) {
            m4[k][hh].x = fmaf(w, v4[k][hh].x, m4[k][hh].x);
            m4[k][hh].y = fmaf(w, v4[k][hh].y, m4[k][hh].y);
            m4[k][hh].z = fmaf(w, v4[k][hh].z, m4[k][hh].z);
            m4[k][hh].w = fmaf(w, v4[k][hh].w, m4[k][hh].w);
          }
        }
    }
    // differentials -> A tile: row 4 bb + s (hi part) and 32 + 4 bb + s (lo part), columns
    // 4 cq .. 4 cq + 3 (8 bytes in the 16-byte unit (cq % 16) / 2 of K chunk cq / 16)
    const int kc = cq >> 4, un = (cq & 15) >> 1, hb = 8 * (cq & 1);
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      const int bb = rb + k;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        if (bb < nb) {
          const float lam = lamv[k][s];
          const float iS = inv_L[5 * bb + 1 + s], iN = inv_L[5 * bb];
          o[0] = m4[k][1 + s].x * iS - lam * (m4[k][0].x * iN);
          o[1] = m4[k][1 + s].y * iS - lam * (m4[k][0].y * iN);
          o[2] = m4[k][1 + s].z * iS - lam * (m4[k][0].z * iN);
          o[3] = m4[k][1 + s].w * iS - lam * (m4[k][0].w * iN);
        }
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          hi[e] = pack_bf162(o[2 * e], o[2 * e + 1]);
          lo[e] = pack_bf162(o[2 * e] - __uint_as_float(hi[e] << 16),
                             o[2 * e + 1] - __uint_as_float(hi[e] & 0xFFFF0000u));
        }
        const int r = 4 * bb + s;
        *reinterpret_cast<uint2*>(smem + A_OFF + kc * A_CHUNK + r * 128 + ((un ^ (r & 7)) << 4) + hb) =
            make_uint2(hi[0], hi[1]);
        *reinterpret_cast<uint2*>(smem + A_OFF + kc * A_CHUNK + (r + 32) * 128 + ((un ^ (r & 7)) << 4) + hb) =
            make_uint2(lo[0], lo[1]);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the gate logits of the CTA's 32 output rows, into the merge-weight area (free now): row
  // r = 4 bb + s, 128 fp32; they land while the MMAs run
  float* G_s = reinterpret_cast<float*>(smem + SCR_OFF);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = 256 * i + tid, r = idx >> 5, c4 = idx & 31, bb = r >> 2;
    if (bb < nb)
      cp_async16(G_s + r * 128 + 4 * c4, p.G + (long long)(b0 + bb) * p.g_ld + (4 * j + (r & 3)) * 128 + 4 * c4);
  }
  const uint32_t tmem = *tmem_slot;
  bool ok = true, issued = false;
  if (tid == 0) {
    ok = mbar_wait(bar_w, 0, ctl, SITE_DEC_MMA);
    if (ok) {
      tc_fence_after();
      issued = true;
      constexpr uint32_t idesc = make_idesc(128, 128, 1, 0, 1);
      const uint64_t da = sdesc_sw128(smem_u32(smem + A_OFF), 16, 1024);
      const uint64_t db = sdesc_sw128(smem_u32(smem + B_OFF), B_NCHUNK, 1024);
#pragma unroll
      for (int kk = 0; kk < 32; ++kk)
        mma_ss(tmem, da + uint64_t((kk >> 2) * (A_CHUNK >> 4) + (kk & 3) * 2), db + uint64_t(kk * 128), idesc,
               kk > 0 ? 1u : 0u);
      mma_commit(bar_mma);
    }
  }
  ok = __syncthreads_and(ok);
  // ---- epilogue.  Warp 0 holds the hi products (TMEM lanes 0..31 = rows 4 bb + s), warp 1 the
  // lo products (lanes 32..63); both park them in the A tile (read by the completed MMAs) as
  // [32 rows][32 float4], float4 c of row r at position c ^ r; then every thread finishes four
  // float4 of the outputs, a warp per 256-byte output row.
  float4* scr = reinterpret_cast<float4*>(smem + A_OFF);     // [2][32][32]
  bool w = ok;
  if (ok && warp < 2) {
    w = __all_sync(0xffffffffu, mbar_wait(bar_mma, 0, ctl, SITE_DEC_MMA));
    tc_fence_after();
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    if (w) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        GDLA_TMEM_LD32(tmem + 32 * c + lane_off, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          scr[(warp * 32 + lane) * 32 + ((8 * c + e) ^ lane)] =
              make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]), __uint_as_float(v[4 * e + 2]),
                          __uint_as_float(v[4 * e + 3]));
      }
    }
  }
  cp_async_wait_all();
  w = __syncthreads_and(w);
  if (w) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = 256 * i + tid, r = idx >> 5, c4 = idx & 31, bb = r >> 2;
      if (bb < nb) {
        const float4 hi = scr[r * 32 + (c4 ^ r)], lo = scr[(32 + r) * 32 + (c4 ^ r)];
        const float4 g = *reinterpret_cast<const float4*>(G_s + r * 128 + 4 * c4);
        const uint2 o = make_uint2(pack_bf162(sigmoidf_fast(g.x) * (hi.x + lo.x), sigmoidf_fast(g.y) * (hi.y + lo.y)),
                                   pack_bf162(sigmoidf_fast(g.z) * (hi.z + lo.z), sigmoidf_fast(g.w) * (hi.w + lo.w)));
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.Dg) + (long long)(b0 + bb) * p.n_signal * 128 +
                                  (4 * j + (r & 3)) * 128 + 4 * c4) = o;
      }
    }
  }
  ok = w;
  if (tid == 0) {
    // before TMEM is released: the MMAs (if issued) are complete, the weight copy has landed
    if (issued) mbar_drain(bar_mma, 0, ctl.err);
    else mbar_drain(bar_w, 0, ctl.err);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

int launch_dec_combine(const DecCombParams& p, KernelCtlHost ctl, cudaStream_t st) {
  if (p.n_ctas > MAXSEG) return -1;
  CUtensorMap mw;
  if (make_tmap_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.W_bKV, (uint64_t)p.n_groups * 256, 512,
                   (uint64_t)p.n_groups * 256 * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  if (cudaFuncSetAttribute(dec_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dcb::SMEM) != cudaSuccess)
    return -4;
  KernelCtl kc{ctl.err, ctl.limit_ns};
  dec_combine_kernel<<<dim3(p.n_groups, (p.B + CB - 1) / CB), 256, dcb::SMEM, st>>>(mw, p, kc);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
