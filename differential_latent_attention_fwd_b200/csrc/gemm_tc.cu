// Projection GEMM on the 5th-generation tensor cores: C[M, N] = A[M, K] * B[K, N].
//
// Used for every linear map of the GDLA layer (picx.dev "Motif 3" summary, section 2.2:
// x W_a^Q, c^Q W_b^Q, x W_a^KV, c W_b^KV, x W^lambda, c^Q W^G and the output projection W^O).
//
// Tiles are 128 x BN.  Warp 0 streams A (K-major, 128-byte swizzle) and B (the [in, out]
// weight: M/N-major, or a [N, K] matrix: K-major) with TMA into a STAGES-deep shared-memory
// ring; one thread of warp 1 issues tcgen05.mma (M = 128, N = BN, K = 16) into a TMEM
// accumulator; the accumulator is drained row-per-thread through the fused epilogue (rotary
// embedding on the rope column range, dtype conversion) and stored.
//
// Products with at least a wave of tiles run persistently: one CTA per SM walks the tiles
// (row tile fastest), with two TMEM accumulators so that four epilogue warps drain tile n
// while the MMA thread already accumulates tile n + 1 and the producer streams tile n + 2's
// operands.  Skinny products (decode, one row tile) run one CTA per tile, optionally with
// K split across CTAs and a reduce kernel that applies the epilogue.
#include "gdla_common.cuh"
#include "gdla_internal.h"

#include <math.h>
#include <string.h>

namespace gdla {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}


// Epilogue of one accumulator row: TMEM columns [0, BN) at t_row -> output row `row`, columns
// n0 .. n0 + BN - 1 (rotary embedding on the rope column range, dtype conversion), or the raw
// fp32 partial of split `split` when ep.partial_out is set.  row_ok = false only drains.
template <int BN>
__device__ __forceinline__ void gemm_epilogue_row(uint32_t t_row, int row, int n0, bool row_ok, int split,
                                                  const GemmEpi& ep) {
  int pos = 0;
  if (ep.rope_hi > ep.rope_lo && row < ep.M) {
    const int dv = ep.pos_div > 1 ? ep.pos_div : 1;
    pos = (ep.pos_ptr ? ep.pos_ptr[row / dv] + row % dv : ((row + ep.row_off) % ep.pos_T)) + ep.pos_off;
  }
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    if (n0 + c0 >= ep.N) break;  // uniform across the warp
    uint32_t r[64];
    GDLA_TMEM_LD32(t_row + c0, r);
    GDLA_TMEM_LD32(t_row + c0 + 32, (r + 32));
    tmem_ld_wait();
    float v[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
    const int col = n0 + c0;
    if (ep.partial_out) {  // split-K pass: raw fp32 partial, epilogue applied by the reduce
      if (row_ok) {
        float* dst = ep.partial_out + ((long long)split * ep.M + row) * ep.N + col;
#pragma unroll
        for (int i = 0; i < 64; i += 4)
          *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
      continue;
    }
    if (col >= ep.rope_lo && col < ep.rope_hi) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float cs, sn;
        rope_cs(pos, ep.rope.inv_freq[i], &cs, &sn);
        const float x1 = v[i], x2 = v[i + 32];
        v[i] = x1 * cs - x2 * sn;
        v[i + 32] = x2 * cs + x1 * sn;
      }
    }
    if (!row_ok) continue;
    const int ncols = min(64, ep.N - col);
    if (ep.out_type == OUT_F32) {
      float* dst = reinterpret_cast<float*>(ep.C) + (long long)row * ep.ldc + col;
      if (ncols == 64) {
#pragma unroll
        for (int i = 0; i < 64; i += 4)
          *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < ncols) dst[i] = v[i];
      }
    } else {
      uint32_t pk[32];
      if (ep.out_type == OUT_BF16) {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf162(v[2 * i], v[2 * i + 1]);
      } else {
        bool bad = false;
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_half2_sat(v[2 * i], v[2 * i + 1], bad);
        if (bad && ep.err) atomicCAS(ep.err, 0, SITE_FP16_RANGE);
      }
      uint16_t* dst = reinterpret_cast<uint16_t*>(ep.C) + (long long)row * ep.ldc + col;
      if (ncols == 64) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(pk[i], pk[i + 1], pk[i + 2], pk[i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < ncols) dst[i] = uint16_t(pk[i >> 1] >> ((i & 1) * 16));
      }
    }
  }
}

// The same epilogue for a whole 128 x BN tile, staged through shared memory (the drained
// operand ring): each thread rounds its accumulator row into a row of the staging tile (16-byte
// pieces at position piece ^ (row % 8)), then the CTA stores whole output rows with
// consecutive threads on consecutive 16-byte pieces.  Needs N % 64 == 0 and 16-byte aligned
// output rows (checked by the launcher).  Called by all 128 threads.
template <int BN>
__device__ __forceinline__ void gemm_epilogue_staged(uint32_t tmem, int m0, int n0, bool ok, int split,
                                                     const GemmEpi& ep, uint8_t* buf, const KernelCtl& ctl) {
  const int t = threadIdx.x, warp = t >> 5;
  const bool f32 = ep.partial_out != nullptr || ep.out_type == OUT_F32;
  const int rowb = f32 ? BN * 4 : BN * 2;              // bytes of a staged row
  const int row = m0 + t;
  // an error raised before this epilogue (not its own fp16 overflow report below) stops the stores
  const bool err_before = *reinterpret_cast<volatile int*>(ctl.err) != 0;
  int pos = 0;
  if (ep.rope_hi > ep.rope_lo && row < ep.M) {
    const int dv = ep.pos_div > 1 ? ep.pos_div : 1;
    pos = (ep.pos_ptr ? ep.pos_ptr[row / dv] + row % dv : ((row + ep.row_off) % ep.pos_T)) + ep.pos_off;
  }
  bool bad = false;
  const uint32_t t_row = tmem + (uint32_t(warp * 32) << 16);
  uint8_t* my = buf + t * rowb;
  const int sw = t & 7;
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    if (n0 + c0 >= ep.N) break;  // uniform
    uint32_t r[64];
    GDLA_TMEM_LD32(t_row + c0, r);
    GDLA_TMEM_LD32(t_row + c0 + 32, (r + 32));
    tmem_ld_wait();
    float v[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
    const int col = n0 + c0;
    if (!ep.partial_out && col >= ep.rope_lo && col < ep.rope_hi) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float cs, sn;
        rope_cs(pos, ep.rope.inv_freq[i], &cs, &sn);
        const float x1 = v[i], x2 = v[i + 32];
        v[i] = x1 * cs - x2 * sn;
        v[i + 32] = x2 * cs + x1 * sn;
      }
    }
    if (f32) {
#pragma unroll
      for (int q = 0; q < 16; ++q)
        *reinterpret_cast<float4*>(my + 16 * ((c0 / 4 + q) ^ sw)) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
      uint32_t pk[32];
      if (ep.out_type == OUT_BF16) {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf162(v[2 * i], v[2 * i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_half2_sat(v[2 * i], v[2 * i + 1], bad);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<uint4*>(my + 16 * ((c0 / 8 + q) ^ sw)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
  // only rows of the product report an fp16 overflow
  if (bad && row < ep.M && ep.err) atomicCAS(ep.err, 0, SITE_FP16_RANGE);
  if (__syncthreads_or(err_before) || !ok) return;
  const int nrows = min(128, ep.M - m0);
  const int ncols = min(BN, ep.N - n0);                 // a multiple of 64
  const int ppr = ncols * (f32 ? 4 : 2) / 16;           // 16-byte pieces of an output row
  uint8_t* base;
  long long ld_bytes;
  if (ep.partial_out) {
    base = reinterpret_cast<uint8_t*>(ep.partial_out + ((long long)split * ep.M + m0) * ep.N + n0);
    ld_bytes = (long long)ep.N * 4;
  } else {
    const int esz = f32 ? 4 : 2;
    base = static_cast<uint8_t*>(ep.C) + ((long long)m0 * ep.ldc + n0) * esz;
    ld_bytes = ep.ldc * esz;
  }
  for (int idx = t; idx < nrows * ppr; idx += 128) {
    const int rr = idx / ppr, q = idx - rr * ppr;
    *reinterpret_cast<uint4*>(base + rr * ld_bytes + 16 * q) =
        *reinterpret_cast<const uint4*>(buf + rr * rowb + 16 * (q ^ (rr & 7)));
  }
}

template <int BN, int STAGES, bool B_KMAJOR>
__global__ void __launch_bounds__(128, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   int K, const __grid_constant__ GemmEpi ep, KernelCtl ctl) {
  constexpr int A_BYTES = 128 * 64 * 2;
  constexpr int B_BYTES = BN * 64 * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN;
  // K blocks of this CTA: all of them, or split blockIdx.z's share (split-K pass)
  const int nk_all = K / 64;
  const int kb0 = ep.kb_per_split > 0 ? int(blockIdx.z) * ep.kb_per_split : 0;
  const int nk = ep.kb_per_split > 0 ? min(ep.kb_per_split, nk_all - kb0) : nk_all;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    uint32_t issued_mask = 0, last_par = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (kb >= STAGES && !mbar_wait(&empty[s], ph ^ 1, ctl, SITE_GEMM_PRODUCER)) break;
      uint8_t* st = smem + s * STAGE;
      mbar_expect_tx(&full[s], STAGE);
      const int kx = (kb0 + kb) * 64;
      tma_load_2d(st, &mapA, &full[s], kx, m0);
      if (B_KMAJOR) {
        tma_load_2d(st + A_BYTES, &mapB, &full[s], kx, n0);
      } else {
#pragma unroll
        for (int c = 0; c < BN / 64; ++c)
          tma_load_2d(st + A_BYTES + c * 8192, &mapB, &full[s], n0 + c * 64, kx);
      }
      issued_mask |= 1u << s;
      last_par = (last_par & ~(1u << s)) | (ph << s);
    }
    // let every copy we issued land before this CTA can retire
    for (int s = 0; s < STAGES; ++s)
      if (issued_mask & (1u << s)) mbar_drain(&full[s], (last_par >> s) & 1, ctl.err);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(128, BN, 1, 0, B_KMAJOR ? 0 : 1);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!mbar_wait(&full[s], ph, ctl, SITE_GEMM_MMA)) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(smem + s * STAGE);
      const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = sdesc_sw128(a_base + k * 32, 16, 1024);
        const uint64_t bd = B_KMAJOR ? sdesc_sw128(b_base + k * 32, 16, 1024)
                                     : sdesc_sw128(b_base + k * 2048, 8192, 1024);
        mma_ss(tmem, ad, bd, idesc, (kb | k) != 0);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  }
  __syncwarp();

  // ---------------- epilogue: thread = accumulator row
  const bool ok = mbar_wait(done, 0, ctl, SITE_GEMM_EPI) || mbar_drain(done, 0, ctl.err);
  tc_fence_after();
  if (ep.staged) {
    // every MMA has completed, so every stage has landed and been read: the ring is free
    gemm_epilogue_staged<BN>(tmem, m0, n0, ok, int(blockIdx.z), ep, smem, ctl);
  } else {
    const int row = m0 + warp * 32 + lane;
    const bool row_ok = ok && row < ep.M && *reinterpret_cast<volatile int*>(ctl.err) == 0;
    gemm_epilogue_row<BN>(tmem + (uint32_t(warp * 32) << 16), row, n0, row_ok, int(blockIdx.z), ep);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, BN);
}

// Persistent form (no split-K): CTA i takes tiles i, i + gridDim.x, ... of the n_m x n_n grid,
// row tile fastest.  Roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-5
// epilogue (warp w drains accumulator rows 32 (w % 4) .. + 31, the TMEM lanes it may access).
template <int BN, int STAGES, bool B_KMAJOR>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_persistent_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                              int K, int n_m, int n_tiles, const __grid_constant__ GemmEpi ep, KernelCtl ctl) {
  constexpr int A_BYTES = 128 * 64 * 2;
  constexpr int B_BYTES = BN * 64 * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;        // [2] accumulator complete (MMA commit)
  uint64_t* acc_empty = acc_full + 2;         // [2] accumulator drained (4 epilogue warps)
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = K / 64;
  const int my_tiles = n_tiles > int(blockIdx.x) ? (n_tiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: k blocks of all this CTA's tiles through one ring
      uint32_t issued_mask = 0, last_par = 0;
      int g = 0;
      bool ok = true;
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int t = int(blockIdx.x) + it * int(gridDim.x);
        const int m0 = (t % n_m) * 128, n0 = (t / n_m) * BN;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (g >= STAGES && !mbar_wait(&empty[s], ph ^ 1, ctl, SITE_GEMM_PRODUCER)) { ok = false; break; }
          uint8_t* st = smem + s * STAGE;
          mbar_expect_tx(&full[s], STAGE);
          const int kx = kb * 64;
          tma_load_2d(st, &mapA, &full[s], kx, m0);
          if (B_KMAJOR) {
            tma_load_2d(st + A_BYTES, &mapB, &full[s], kx, n0);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(st + A_BYTES + c * 8192, &mapB, &full[s], n0 + c * 64, kx);
          }
          issued_mask |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
        }
      }
      // let every copy we issued land before this CTA can retire
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) mbar_drain(&full[s], (last_par >> s) & 1, ctl.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: accumulator it & 1 for this CTA's tile it
      constexpr uint32_t idesc = make_idesc(128, BN, 1, 0, B_KMAJOR ? 0 : 1);
      int g = 0;
      bool ok = true;
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int a = it & 1;
        if (it >= 2 && !mbar_wait(&acc_empty[a], ((it >> 1) - 1) & 1, ctl, SITE_GEMM_MMA)) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(a * BN);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, ctl, SITE_GEMM_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * STAGE);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bd = B_KMAJOR ? sdesc_sw128(b_base + k * 32, 16, 1024)
                                         : sdesc_sw128(b_base + k * 2048, 8192, 1024);
            mma_ss(d, ad, bd, idesc, (kb | k) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[a]);
      }
      // every MMA has completed before TMEM is released
      mma_commit(done);
      mbar_drain(done, 0, ctl.err);
    }
  } else {
    // ---------------- epilogue warps 2-5: thread = accumulator row
    const int q = warp & 3;
    for (int it = 0; it < my_tiles; ++it) {
      const int a = it & 1;
      bool ok = mbar_wait(&acc_full[a], (it >> 1) & 1, ctl, SITE_GEMM_EPI);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int t = int(blockIdx.x) + it * int(gridDim.x);
      const int m0 = (t % n_m) * 128, n0 = (t / n_m) * BN;
      const int row = m0 + q * 32 + lane;
      const bool row_ok = row < ep.M && *reinterpret_cast<volatile int*>(ctl.err) == 0;
      gemm_epilogue_row<BN>(tmem + uint32_t(a * BN) + (uint32_t(q * 32) << 16), row, n0, row_ok, 0, ep);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// Split-K reduce: out = epilogue(sum over splits).  Thread = column pair (i, i + 32) of a
// 64-column block, so that rope pairs stay in one thread.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const __grid_constant__ GemmEpi ep, int splits) {
  const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int nblk = ep.N / 64;
  if (idx >= (long long)ep.M * nblk * 32) return;
  const int i = int(idx & 31);
  const int blk = int((idx >> 5) % nblk);
  const int row = int((idx >> 5) / nblk);
  const int c1 = blk * 64 + i, c2 = c1 + 32;
  float a = 0.f, b = 0.f;
  for (int z = 0; z < splits; ++z) {
    const float* pz = ep.splitk + ((long long)z * ep.M + row) * ep.N;
    a += pz[c1];
    b += pz[c2];
  }
  if (blk * 64 >= ep.rope_lo && blk * 64 < ep.rope_hi) {
    const int dv = ep.pos_div > 1 ? ep.pos_div : 1;
    const int pos = (ep.pos_ptr ? ep.pos_ptr[row / dv] + row % dv : ((row + ep.row_off) % ep.pos_T)) + ep.pos_off;
    float cs, sn;
    rope_cs(pos, ep.rope.inv_freq[i], &cs, &sn);
    const float x1 = a, x2 = b;
    a = x1 * cs - x2 * sn;
    b = x2 * cs + x1 * sn;
  }
  const long long o = (long long)row * ep.ldc;
  if (ep.out_type == OUT_F32) {
    reinterpret_cast<float*>(ep.C)[o + c1] = a;
    reinterpret_cast<float*>(ep.C)[o + c2] = b;
  } else if (ep.out_type == OUT_BF16) {
    reinterpret_cast<__nv_bfloat16*>(ep.C)[o + c1] = __float2bfloat16_rn(a);
    reinterpret_cast<__nv_bfloat16*>(ep.C)[o + c2] = __float2bfloat16_rn(b);
  } else {
    bool bad = false;
    reinterpret_cast<__half*>(ep.C)[o + c1] = half_sat(a, bad);
    reinterpret_cast<__half*>(ep.C)[o + c2] = half_sat(b, bad);
    if (bad && ep.err) atomicCAS(ep.err, 0, SITE_FP16_RANGE);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                 CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return -1;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -2;
}

void fill_rope_table(RopeTable* t, int d_rope, double theta) {
  memset(t, 0, sizeof(*t));
  t->d_rope = d_rope;
  for (int i = 0; i < d_rope / 2 && i < 32; ++i) t->inv_freq[i] = pow(theta, -2.0 * i / d_rope);
}

// SMs of the current device (queried once per device).
static int g_num_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cached[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  }
  return cached[dev];
}

template <int BN, int STAGES, bool BK>
static int run_gemm(const CUtensorMap& ma, const CUtensorMap& mb, int M, int N, int K,
                    const GemmEpi& ep, KernelCtlHost ctl, cudaStream_t st, int splits) {
  constexpr int STAGE = 128 * 64 * 2 + BN * 64 * 2;
  const int smem = STAGES * STAGE + 1024 + 256;
  auto kfn = gemm_tc_kernel<BN, STAGES, BK>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return -4;
  KernelCtl kc{ctl.err, ctl.limit_ns};
  const int n_m = (M + 127) / 128, n_n = (N + BN - 1) / BN;
  if (splits == 1 && (long long)n_m * n_n >= 2 * g_num_sms()) {
    auto pfn = gemm_tc_persistent_kernel<BN, STAGES, BK>;
    const int psmem = STAGES * STAGE + 1024 + 256;
    if (cudaFuncSetAttribute(pfn, cudaFuncAttributeMaxDynamicSharedMemorySize, psmem) != cudaSuccess)
      return -4;
    const int n_tiles = n_m * n_n;
    const int ctas = n_tiles < g_num_sms() ? n_tiles : g_num_sms();
    pfn<<<ctas, 192, psmem, st>>>(ma, mb, K, n_m, n_tiles, ep, kc);
    return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
  }
  dim3 grid(n_m, n_n, splits);
  kfn<<<grid, 128, smem, st>>>(ma, mb, K, ep, kc);
  if (cudaPeekAtLastError() != cudaSuccess) return -4;
  if (splits > 1) {
    const long long threads = (long long)M * (N / 64) * 32;
    splitk_reduce_kernel<<<unsigned((threads + 255) / 256), 256, 0, st>>>(ep, splits);
    if (cudaPeekAtLastError() != cudaSuccess) return -4;
    count_extra_launch();
  }
  return 0;
}

static int gemm_bn(int N) { return N >= 256 ? 256 : (N > 64 ? 128 : 64); }

// Skinny products (one 128-row M tile) leave most SMs idle; split K so that the CTAs streaming
// the weights fill at most one wave, each split keeping at least 4 K blocks of 64.
int gemm_splitk_count(int M, int N, int K) {
  if (M > 128 || N % 64 != 0 || K % 64 != 0) return 1;
  const int BN = gemm_bn(N);
  const int tiles = (N + BN - 1) / BN;
  const int nk = K / 64;
  int s = g_num_sms() / tiles;
  s = s > nk / 4 ? nk / 4 : s;
  if (s <= 1) return 1;
  const int kps = (nk + s - 1) / s;
  return (nk + kps - 1) / kps;
}

int launch_gemm(const void* A, long long lda, const void* B, long long ldb, bool b_kmajor, int M,
                int N, int K, const GemmEpi& ep_in, KernelCtlHost ctl, cudaStream_t st) {
  if (M <= 0 || N <= 0) return 0;
  if (K <= 0 || K % 64 != 0) return -1;
  const int BN = gemm_bn(N);
  GemmEpi ep = ep_in;
  ep.err = ctl.err;
  ep.partial_out = nullptr;
  ep.kb_per_split = 0;
  int splits = 1;
  if (ep.splitk) {
    splits = gemm_splitk_count(M, N, K);
    if ((long long)splits * M * N > ep.splitk_floats) splits = 1;
    if (splits > 1) {
      const int nk = K / 64;
      ep.kb_per_split = (nk + splits - 1) / splits;
      ep.partial_out = ep.splitk;
    }
  }
  {
    // the staged epilogue of the one-tile kernel: whole 64-column chunks, 16-byte aligned rows
    const bool f32 = ep.partial_out != nullptr || ep.out_type == OUT_F32;
    const int esz = f32 ? 4 : 2;
    const uintptr_t cb = ep.partial_out ? reinterpret_cast<uintptr_t>(ep.partial_out) : reinterpret_cast<uintptr_t>(ep.C);
    const long long ldb_out = ep.partial_out ? (long long)N * 4 : ep.ldc * esz;
    ep.staged = N % 64 == 0 && cb % 16 == 0 && ldb_out % 16 == 0;
  }
  CUtensorMap ma, mb;
  if (make_tmap_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, M, lda * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  int rc;
  if (b_kmajor)
    rc = make_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, N, ldb * 2, 64, BN,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  else
    rc = make_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, K, ldb * 2, 64, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return -3;
  if (b_kmajor) {
    if (BN == 256) return run_gemm<256, 4, true>(ma, mb, M, N, K, ep, ctl, st, splits);
    if (BN == 128) return run_gemm<128, 6, true>(ma, mb, M, N, K, ep, ctl, st, splits);
    return run_gemm<64, 8, true>(ma, mb, M, N, K, ep, ctl, st, splits);
  }
  if (BN == 256) return run_gemm<256, 4, false>(ma, mb, M, N, K, ep, ctl, st, splits);
  if (BN == 128) return run_gemm<128, 6, false>(ma, mb, M, N, K, ep, ctl, st, splits);
  return run_gemm<64, 8, false>(ma, mb, M, N, K, ep, ctl, st, splits);
}

}  // namespace gdla
