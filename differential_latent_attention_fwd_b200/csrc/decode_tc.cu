// Absorbed-form GDLA decode attention on the tensor cores (sm_100a).
//
// For one sequence b the 80 query heads all attend over the same latent-cache rows
// c_p = [c_bar_p (512) | rotated k^R_p (64)] (the MLA weight absorption: q~_h = [W_UK q^C_h ; q^R_h],
// score_{h,p} = q~_h . c_p / sqrt(192); picx.dev Motif 3 summary, section 2.2, with K and V
// regrouped into the latent space).  A CTA owns one (sequence, split of the key range) and
// computes, per 128-position tile and with positions on the 128 TMEM lanes ("swap AB"):
//   S^T[p, h]   = C[p, :] . q~[h, :]            tcgen05.mma M 128 (positions), N 80, K 576
//   P[p, h]     = 2^(S^T log2e/sqrt(192) - m_h)  (softmax numerators, bf16, in shared memory)
//   O^T[l, h]  += C[:, l]^T P[:, h]              4 x tcgen05.mma M 128 (latent rows), N 80, K 128
// and finally writes the split's partial (O^T, m_h, sum_p P) for the merge kernel.
//
// Shared memory cannot hold q~ (80 x 576 bf16 = 90 KB) together with a whole 128-position tile
// (144 KB), so the tile's latent columns are fetched twice: once with the rope columns for the
// scores, and again for the PV product right after (an L2 hit).  The TMA ring has three 32 KB
// slots, each holding a pair of 64-column boxes (the two halves of one 128-row M block of C^T).
// The running maximum m_h moves only when a score exceeds it by more than 2^8 (then O^T and the
// per-position partial sums are rescaled), which is exact after the final division.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-5 softmax
// (thread = position = TMEM lane; later thread = latent row for the O^T read-out).
#include "gdla_common.cuh"
#include "gdla_decode.h"
#include "gdla_internal.h"

namespace gdla {

namespace dtc {
constexpr int NH = 80;
constexpr int SLOT = 32768;
constexpr int NSLOT = 3;
constexpr int QBOX = NH * 128;                 // one [80 rows][64 bf16] box of q~
constexpr int RING_OFF = 0;
constexpr int QT_OFF = NSLOT * SLOT;           // 9 boxes of q~
constexpr int P_OFF = QT_OFF + 9 * QBOX;       // P^T: [80 heads][128 positions] as 2 K-chunks
constexpr int BAR_OFF = P_OFF + 2 * QBOX;
constexpr int SMEM = BAR_OFF + 2048 + 1024;
constexpr int S_COL0 = 0, S_COL1 = 96, O_COL = 192;   // TMEM columns
constexpr float RESCALE_THRESHOLD = 8.0f;
}  // namespace dtc

struct DecBars {
  float m_ref[dtc::NH];        // reference maxima (log2 units), 16-byte aligned for float4 reads
  float red[4][dtc::NH];       // cross-warp reduction scratch
  uint64_t q_full;
  uint64_t ring_full[dtc::NSLOT], ring_empty[dtc::NSLOT];
  uint64_t s_full[2], p_ready, pv_done, mma_final;
  uint32_t tmem_base;
};

__device__ __forceinline__ uint8_t* dtc_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Key tiles [t_begin, t_end) of this split and the sequence's valid key range [lo, hi].
struct DecRange {
  int lo, hi, t_begin, t_end;
};
__device__ __forceinline__ DecRange dec_range(const DecAttnParams& p, int b, int sp, int* err) {
  DecRange r;
  // row b is new token b % q_len of its sequence: it sees the cached keys and the new tokens
  // up to itself, all held in the cache rows 0 .. cache_len + b % q_len
  const int ql = p.q_len > 1 ? p.q_len : 1;
  const int L0 = p.cache_len[b / ql];
  int L = L0 + b % ql;
  if (L0 < 0 || L0 + ql - 1 >= p.cap) {
    if (threadIdx.x == 0) atomicCAS(err, 0, SITE_BAD_CACHE_LEN);
    r.lo = 0; r.hi = -1; r.t_begin = 0; r.t_end = 0;
    return r;
  }
  r.hi = L;
  r.lo = p.window > 0 ? max(0, L - p.window + 1) : 0;
  const int t0 = r.lo / 128, t1 = r.hi / 128 + 1;
  const int per = (t1 - t0 + p.n_split - 1) / p.n_split;
  r.t_begin = min(t1, t0 + sp * per);
  r.t_end = min(t1, r.t_begin + per);
  return r;
}

__global__ void __launch_bounds__(192, 1)
    dec_attn_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapC,
                       const __grid_constant__ DecAttnParams p, KernelCtl ctl) {
  using namespace dtc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = dtc_align(smem_raw);
  DecBars* bars = reinterpret_cast<DecBars*>(smem + BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sp = blockIdx.x, b = blockIdx.y;
  const DecRange rg = dec_range(p, b, sp, ctl.err);
  const int n_t = rg.t_end - rg.t_begin;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&bars->ring_full[s], 1);
      mbar_init(&bars->ring_empty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_ready, 128);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->mma_final, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapC);
  }
  if (threadIdx.x < NH) bars->m_ref[threadIdx.x] = -INFINITY;
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const long long crow0 = (long long)(b / (p.q_len > 1 ? p.q_len : 1)) * p.cap;

  if (warp == 0) {
    if (lane == 0 && n_t > 0) {
      // ============================================================ TMA producer
      uint32_t issued = 0, par = 0;
      bool ok = true;
      mbar_expect_tx(&bars->q_full, 9 * QBOX);
      for (int c = 0; c < 9; ++c)
        tma_load_2d(smem + QT_OFF + c * QBOX, &mapQ, &bars->q_full, c * 64, b * NH);
      uint32_t g = 0;
      // The latent columns are read twice (scores, then PV): the first read asks L2 to keep
      // them, the second (and the rope columns, read once) lets them go.
      const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
      // unit order: S(0), S(1), P(0), S(2), P(1), ..., S(n-1), P(n-2), P(n-1)
      auto load_unit = [&](int tile, int pair, bool rope, bool second) -> bool {
        const int slot = g % NSLOT;
        const uint32_t ph = (g / NSLOT) & 1;
        if (g >= NSLOT && !mbar_wait(&bars->ring_empty[slot], ph ^ 1, ctl, SITE_DEC_PRODUCER))
          return false;
        uint8_t* dst = smem + RING_OFF + slot * SLOT;
        const int y = int(crow0 + (long long)(rg.t_begin + tile) * 128);
        if (rope) {
          mbar_expect_tx(&bars->ring_full[slot], 16384);
          tma_load_2d_hint(dst, &mapC, &bars->ring_full[slot], 512, y, drop);
        } else {
          const uint64_t pol = second ? drop : keep;
          mbar_expect_tx(&bars->ring_full[slot], 32768);
          tma_load_2d_hint(dst, &mapC, &bars->ring_full[slot], pair * 128, y, pol);
          tma_load_2d_hint(dst + 16384, &mapC, &bars->ring_full[slot], pair * 128 + 64, y, pol);
        }
        issued |= 1u << slot;
        par = (par & ~(1u << slot)) | (ph << slot);
        ++g;
        return true;
      };
      for (int i = 0; i <= n_t && ok; ++i) {
        if (i < n_t)
          for (int u = 0; u < 5 && ok; ++u) ok = load_unit(i, u, u == 4, false);
        if (i >= 1)
          for (int u = 0; u < 4 && ok; ++u) ok = load_unit(i - 1, u, false, true);
      }
      for (int s = 0; s < NSLOT; ++s)
        if (issued & (1u << s)) mbar_drain(&bars->ring_full[s], (par >> s) & 1, ctl.err);
      mbar_drain(&bars->q_full, 0, ctl.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_t > 0) {
      // ============================================================ MMA issuer
      constexpr uint32_t idesc_s = make_idesc(128, NH, 1, 0, 0);
      constexpr uint32_t idesc_o = make_idesc(128, NH, 1, 1, 0);
      const uint32_t ring = smem_u32(smem + RING_OFF);
      const uint32_t qt = smem_u32(smem + QT_OFF);
      const uint32_t pt = smem_u32(smem + P_OFF);
      uint32_t g = 0, pr_par = 0;
      bool ok = mbar_wait(&bars->q_full, 0, ctl, SITE_DEC_MMA);
      // ring units are consumed strictly in load order, one at a time: wait, issue, release
      auto wait_unit = [&]() -> bool {
        if (!mbar_wait(&bars->ring_full[g % NSLOT], (g / NSLOT) & 1, ctl, SITE_DEC_MMA)) return false;
        tc_fence_after();
        return true;
      };
      auto release_unit = [&]() {
        mma_commit(&bars->ring_empty[g % NSLOT]);
        ++g;
      };
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(&bars->p_ready, pr_par, ctl, SITE_DEC_MMA)) return false;
        pr_par ^= 1;
        tc_fence_after();
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          if (!wait_unit()) return false;
          const uint32_t a0 = ring + (g % NSLOT) * SLOT;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = sdesc_sw128(a0 + kk * 2048, 16384, 1024);
            const uint64_t bd = sdesc_sw128(pt + (kk >> 2) * QBOX + (kk & 3) * 32, 16, 1024);
            mma_ss(tmem + O_COL + NH * mb, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          release_unit();
        }
        mma_commit(&bars->pv_done);
        return true;
      };
      for (int i = 0; i < n_t && ok; ++i) {
        // ---- S^T(i) = C(i) q~^T into S buffer i & 1, one ring unit (64-col box pair) at a time
        const uint32_t d = tmem + ((i & 1) ? S_COL1 : S_COL0);
#pragma unroll 1
        for (int u = 0; u < 5 && ok; ++u) {
          if (!wait_unit()) { ok = false; break; }
          const uint32_t slot = ring + (g % NSLOT) * SLOT;
          const int nbox = u < 4 ? 2 : 1;
          for (int bx = 0; bx < nbox; ++bx) {
            const int c = u < 4 ? 2 * u + bx : 8;    // K chunk: latent 0..7, rope 8
            const uint32_t a0 = slot + bx * 16384;
            const uint32_t b0 = qt + c * QBOX;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(d, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                     idesc_s, (c | kk) != 0);
          }
          release_unit();
        }
        if (!ok) break;
        mma_commit(&bars->s_full[i & 1]);
        // ---- O^T += C(i-1)^T P(i-1)
        if (i >= 1 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_t - 1);
      mma_commit(&bars->mma_final);
      mbar_drain(&bars->mma_final, 0, ctl.err);
    }
  } else {
    // ============================================================ softmax (warps 2..5)
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int r = q * 32 + lane;            // position within the tile / latent row
    const int tw = threadIdx.x - 64;        // 0..127 inside the softmax group
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    float l_part[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) l_part[h] = 0.f;
    uint32_t s_par[2] = {0, 0};
    int pv_seen = 0;                        // PVs known complete
    bool ok = true;
    auto wait_pv = [&](int k) -> bool {     // wait until PV(k) has completed
      if (pv_seen > k) return true;
      bool w = mbar_wait(&bars->pv_done, k & 1, ctl, SITE_DEC_SOFTMAX);
      w = __all_sync(0xffffffffu, w);
      if (w) pv_seen = k + 1;
      return w;
    };
    uint8_t* P = smem + P_OFF;
    // Every outcome of a bounded wait is made uniform over the 128 softmax threads before it
    // steers control flow, so that no thread is left alone at a named barrier.
    auto group_ok = [&](bool w) { return !named_bar_or(1, 128, !w); };
    for (int i = 0; i < n_t && ok; ++i) {
      const int buf = i & 1;
      const bool w = mbar_wait(&bars->s_full[buf], s_par[buf], ctl, SITE_DEC_SOFTMAX);
      if (!group_ok(w)) { ok = false; break; }
      s_par[buf] ^= 1;
      tc_fence_after();
      const uint32_t tS = tmem + (buf ? S_COL1 : S_COL0) + lane_off;
      const int pos = (rg.t_begin + i) * 128 + r;
      const bool valid = pos >= rg.lo && pos <= rg.hi;
      // scores are re-read from TMEM in 16-head chunks: (log2-scaled) score of head 16c + e
      auto load_chunk = [&](int c, float* v) {
        uint32_t u[16];
        GDLA_TMEM_LD16(tS + 16 * c, u);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = valid ? __uint_as_float(u[e]) * p.scale_log2 : -INFINITY;
      };
      bool above = false;
#pragma unroll 1
      for (int c = 0; c < 5; ++c) {
        float v[16];
        load_chunk(c, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) above |= v[e] > bars->m_ref[16 * c + e] + RESCALE_THRESHOLD;
      }
      if (named_bar_or(1, 128, above)) {
        // exact per-head maximum of this tile, then move the reference maxima
#pragma unroll 1
        for (int c = 0; c < 5; ++c) {
          float v[16];
          load_chunk(c, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x = v[e];
#pragma unroll
            for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
            if (lane == ((16 * c + e) & 31)) bars->red[q][16 * c + e] = x;
          }
        }
        named_bar_sync(1, 128);
        if (tw < NH) {
          const float tmax = fmaxf(fmaxf(bars->red[0][tw], bars->red[1][tw]),
                                   fmaxf(bars->red[2][tw], bars->red[3][tw]));
          const float mo = bars->m_ref[tw];
          const float mn = fmaxf(mo, tmax);
          bars->red[0][tw] = mn == -INFINITY ? 1.f : ex2_approx(mo - mn);   // scale of old terms
          bars->red[1][tw] = mn;
        }
        named_bar_sync(1, 128);
#pragma unroll
        for (int h = 0; h < NH; ++h) l_part[h] *= bars->red[0][h];
        if (i > 0) {
          // O^T must hold PV(0..i-1) before it is rescaled
          if (!group_ok(wait_pv(i - 1))) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4 * 5; ++c) {          // 4 M blocks x 5 chunks of 16 heads
            const uint32_t tO = tmem + O_COL + NH * (c / 5) + 16 * (c % 5) + lane_off;
            uint32_t o[16];
            GDLA_TMEM_LD16(tO, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              o[e] = __float_as_uint(__uint_as_float(o[e]) * bars->red[0][16 * (c % 5) + e]);
            GDLA_TMEM_ST16(tO, o);
          }
          tmem_st_wait();
        }
        named_bar_sync(1, 128);
        if (tw < NH) bars->m_ref[tw] = bars->red[1][tw];
        named_bar_sync(1, 128);
      }
      // the single P buffer is free once PV(i-1) has completed
      if (i > 0 && !group_ok(wait_pv(i - 1))) { ok = false; break; }
      {
        // numerators of this tile, rounded to bf16 (the row sums use the rounded values)
        const int chunk = r >> 6, pc = r & 63;
        uint8_t* base = P + chunk * QBOX + ((pc & 7) << 1);
#pragma unroll
        for (int c = 0; c < 5; ++c) {
          float v[16];
          load_chunk(c, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int hh = 16 * c + e;
            const float mr = bars->m_ref[hh];
            const float mu = mr == -INFINITY ? 0.f : mr;
            const __nv_bfloat16 pbv = __float2bfloat16_rn(ex2_approx(v[e] - mu));
            l_part[hh] += __bfloat162float(pbv);
            *reinterpret_cast<__nv_bfloat16*>(base + hh * 128 + ((((pc >> 3) ^ (hh & 7))) << 4)) = pbv;
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_ready);
    }
    // ---------------- split partials
    if (ok && n_t > 0 && !group_ok(wait_pv(n_t - 1))) ok = false;
    tc_fence_after();
    // row sums: per head, over the 128 positions
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float v = l_part[h];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == (h & 31)) bars->red[q][h] = v;
    }
    named_bar_sync(1, 128);
    const long long pbase = ((long long)b * p.n_split + sp) * NH;
    if (tw < NH) {
      float* ml = p.ml + (pbase + tw) * 2;
      const float lsum = bars->red[0][tw] + bars->red[1][tw] + bars->red[2][tw] + bars->red[3][tw];
      ml[0] = bars->m_ref[tw];
      ml[1] = (ok && n_t > 0) ? lsum : 0.f;
    }
    if (ok && n_t > 0) {
#pragma unroll 1
      for (int mb = 0; mb < 4; ++mb) {
        const uint32_t tO = tmem + O_COL + NH * mb + lane_off;
        uint32_t o[NH];
        GDLA_TMEM_LD32(tO, o);
        GDLA_TMEM_LD32(tO + 32, (o + 32));
        GDLA_TMEM_LD16(tO + 64, (o + 64));
        tmem_ld_wait();
        float* dst = p.part + pbase * 512 + 128 * mb + r;
#pragma unroll
        for (int h = 0; h < NH; ++h) dst[(long long)h * 512] = __uint_as_float(o[h]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int launch_dec_attn_tc(const DecAttnParams& p, KernelCtlHost ctl, cudaStream_t st) {
  CUtensorMap mq, mc;
  if (make_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.qt, 576, (uint64_t)p.B * dtc::NH, 576 * 2,
                   64, dtc::NH, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.cache, 576, (uint64_t)p.B * p.cap, 576 * 2,
                   64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  if (cudaFuncSetAttribute(dec_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           dtc::SMEM) != cudaSuccess)
    return -4;
  dim3 grid(p.n_split, p.B);
  KernelCtl kc{ctl.err, ctl.limit_ns};
  dec_attn_tc_kernel<<<grid, 192, dtc::SMEM, st>>>(mq, mc, p, kc);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// Number of key-range splits per sequence: minimises (waves of 148 CTAs) x (tiles per split + 2),
// the +2 standing for the per-CTA set-up and drain.
int decode_split_count(int B, int cap, int window) {
  const int keys = window > 0 ? (window < cap ? window : cap) : cap;
  const int tiles = (keys + 127) / 128 + 1;
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= 64; ++s) {
    const long long waves = ((long long)B * s + 147) / 148;
    const long long cost = waves * ((tiles + s - 1) / s + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

}  // namespace gdla
