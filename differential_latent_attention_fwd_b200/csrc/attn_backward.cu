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
//
// Every contraction runs on the 5th-generation tensor cores (tcgen05, fp16 operands, fp32
// accumulators in TMEM), in two kernels that each own their outputs (no atomics):
//  * keys stationary (dK, dV): one CTA per (sequence, KV group j, 128 keys) keeps K = [K^C_j |
//    k^R] and V_j of its keys in shared memory and loops over 64-query tiles x the group's five
//    heads: S^T = K q^T and dP^T = V dH^T into TMEM; the elementwise threads (EL_GROUPS per key,
//    each taking QG of the 64 queries) turn them into P^T and dS'^T (fp16, packed into the S^T
//    slot, each thread over the columns it has read) which are the A operands of
//    dV += P^T dH and dK += dS'^T q.  TMEM: three rotating 64-column slots | dV 128 | dK 192.
//    Unit u puts S^T in slot u % 3 and dP^T in slot (u + 1) % 3; the dP^T slot is free as soon
//    as the elementwise threads have read it, so the tensor core computes S^T / dP^T of unit
//    u + 1 (and dV / dK of unit u - 1) while they work on unit u.
//  * queries stationary (dq): one CTA per (sequence, head, 128 queries) keeps q and dH and loops
//    over 64-key tiles: S = q K^T, dP = dH V^T, dS' in place (EL_GROUPS threads per query, QG
//    keys each), dq += dS' K.
//    TMEM: two (S 64 | dP 64) buffers | dq 192 columns, so that the scores of the next key tile
//    are computed while the elementwise threads work on this one.
// Both recompute P from the saved log-sum-exp; the second recomputes S and dP, which costs
// 1152 instead of the minimal 832 multiply-adds per (query, key, head) but needs neither a
// materialised score matrix nor dq accumulation across CTAs.  dk^R is the sum over the 16 KV
// groups of their rotary parts (a small reduce at the end).
#include "gdla_common.cuh"
#include "gdla_internal.h"

namespace gdla {

namespace bwd {
constexpr int BK = 128;   // keys per dK/dV CTA (TMEM lanes)
constexpr int BQ = 128;   // queries per dq CTA (TMEM lanes)
constexpr int TQ = 64;    // query tile of the dK/dV loop
constexpr int TK = 64;    // key tile of the dq loop
constexpr int NST = 3;    // stages of the streamed operand ring
// elementwise threads per key (dK/dV) or query (dq): group e of warps 2 + 4 e .. 5 + 4 e takes
// the QG queries (keys) QG e .. QG e + QG - 1 of a 64-wide tile
constexpr int EL_GROUPS = 4;
constexpr int QG = 64 / EL_GROUPS;
constexpr int EL_WARPS = 4 * EL_GROUPS;
constexpr int THREADS = 64 + 32 * EL_WARPS;
constexpr int BOX_BIG = 128 * 128;    // [128 rows][64 fp16] 128-byte-swizzled box
constexpr int BOX_SMALL = 64 * 128;   // [64 rows][64 fp16]
// dK/dV kernel: K block (3 boxes) | V block (2) | ring of (q tile 3 boxes + dH tile 2 boxes) |
// per-warp lse/Delta staging | barriers
constexpr int A_K_OFF = 0;
constexpr int A_V_OFF = A_K_OFF + 3 * BOX_BIG;
constexpr int A_RING = A_V_OFF + 2 * BOX_BIG;
constexpr int STAGE = 5 * BOX_SMALL;
constexpr int A_LD_OFF = A_RING + NST * STAGE;
constexpr int A_BAR_OFF = A_LD_OFF + EL_WARPS * 2 * QG * 4;
constexpr int A_SMEM = A_BAR_OFF + 256 + 1024;
// dq kernel: q block (3 boxes) | dH block (2) | ring of (K tile 3 boxes + V tile 2 boxes)
constexpr int B_Q_OFF = 0;
constexpr int B_H_OFF = B_Q_OFF + 3 * BOX_BIG;
constexpr int B_RING = B_H_OFF + 2 * BOX_BIG;
constexpr int B_BAR_OFF = B_RING + NST * STAGE;
constexpr int B_SMEM = B_BAR_OFF + 256 + 1024;
constexpr int T_S = 0, T_DP = 64;                // dq kernel: S / dP buffers at 0 (+64) and 128 (+64),
constexpr int T_DQ = 256;                        // dq at 256
constexpr int T_DV = 192, T_DK = 320;            // dK/dV kernel: slots at 0, 64, 128
static_assert(A_SMEM <= 232448 && B_SMEM <= 232448, "shared memory");
}  // namespace bwd

struct BwdBars {
  uint64_t fixed_full;                      // the CTA's stationary block (K, V or q, dH)
  uint64_t full[bwd::NST], empty[bwd::NST];
  uint64_t s_full, p_ready, acc_done, mma_final;
  uint64_t s_full2[2], p_ready2[2], buf_free2[2];   // the dq kernel's two S / dP buffers
  uint64_t el_read, dvdk_done;                      // the dK/dV kernel's slot rotation
  uint32_t tmem_base;
};

struct BwdTcParams {
  int B, T, window, n_signal, n_groups, Tpad;
  long long M;
  float scale_log2, scale;
  const float* lseT;    // [n_heads][B][Tpad]: log2-sum-exp2 of the scaled scores
  const float* deltaT;  // [n_heads][B][Tpad]: Delta = rowsum(dH H)
  float* dK;            // [M][n_groups][192]: d[K^C_j | k^R] of group j (dK/dV kernel)
  float* d_kv;          // [M][n_groups * 256]: dV into the V columns (dK/dV kernel)
  float* d_qq;          // [M][n_heads * 192] in the QQ column layout (dq kernel)
};

__device__ __forceinline__ uint8_t* bwd_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// Head of KV group j at slot i of the group: 0 = the noise head, 1..g = the signal heads.
__device__ __forceinline__ int head_of(int i, int j, int n_signal, int g) {
  return i == 0 ? n_signal + j : g * j + i - 1;
}
// Is query t allowed to see key s (causal, window W; both inside the sequence)?
// The elementwise group's QG columns (32 lanes) out of TMEM, and half as many back.
__device__ __forceinline__ void el_tmem_ld(uint32_t taddr, uint32_t* r) {
  if constexpr (bwd::QG == 32) {
    GDLA_TMEM_LD32(taddr, r);
  } else {
    static_assert(bwd::QG == 16, "elementwise group width");
    GDLA_TMEM_LD16(taddr, r);
  }
}
__device__ __forceinline__ void el_tmem_st_half(uint32_t taddr, const uint32_t* r) {
  if constexpr (bwd::QG == 32) {
    GDLA_TMEM_ST16(taddr, r);
  } else {
    GDLA_TMEM_ST8(taddr, r);
  }
}
// First TMEM column of the fp16 pairs of queries (keys) 16 kk .. 16 kk + 15, written by
// elementwise group 16 kk / QG at the start of its QG columns.
__device__ __forceinline__ constexpr uint32_t el_col(int kk) {
  return uint32_t(bwd::QG * ((16 * kk) / bwd::QG) + ((16 * kk) % bwd::QG) / 2);
}
__device__ __forceinline__ bool bwd_visible(int t, int s, int T, int W) {
  return t < T && s <= t && (W <= 0 || t - s < W);
}

__device__ __forceinline__ void bwd_init_bars(BwdBars* bars, uint32_t n_el_warps) {
  mbar_init(&bars->fixed_full, 1);
  for (int s = 0; s < bwd::NST; ++s) {
    mbar_init(&bars->full[s], 1);
    mbar_init(&bars->empty[s], 1);
  }
  mbar_init(&bars->s_full, 1);
  mbar_init(&bars->p_ready, n_el_warps);     // one arrival per elementwise warp
  mbar_init(&bars->acc_done, 1);
  mbar_init(&bars->mma_final, 1);
  mbar_init(&bars->el_read, n_el_warps);     // one arrival per elementwise warp: dP^T read
  mbar_init(&bars->dvdk_done, 1);
  for (int i = 0; i < 2; ++i) {
    mbar_init(&bars->s_full2[i], 1);
    mbar_init(&bars->p_ready2[i], n_el_warps);
    mbar_init(&bars->buf_free2[i], 1);
  }
  fence_mbar_init();
}

// =================================================================== keys stationary: dK, dV
// Grid (KV group, key block, sequence): the heaviest causal blocks (first keys) launch first.
// Roles (THREADS threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2 .. 1 +
// EL_WARPS elementwise: EL_GROUPS threads per key (TMEM lane 32 (warp % 4) + lane), group e
// (warps 2 + 4 e .. 5 + 4 e) taking the queries QG e .. QG e + QG - 1 of a unit, so that the
// elementwise step of a unit, which the tensor core waits for, is split EL_GROUPS ways.
__global__ void __launch_bounds__(bwd::THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                    const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mH,
                    const __grid_constant__ BwdTcParams p, KernelCtl ctl) {
  using namespace bwd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = bwd_align(smem_raw);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + A_BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x, kb = blockIdx.y, b = blockIdx.z;
  const int g = p.n_signal / p.n_groups;
  const int k0 = kb * BK;
  const int q_begin = (k0 / TQ) * TQ;
  const int q_end = p.window > 0 ? min(p.T, k0 + BK - 1 + p.window) : p.T;
  const int n_tiles = q_end > q_begin ? (q_end - q_begin + TQ - 1) / TQ : 0;
  const int n_units = n_tiles * (g + 1);      // unit u: query tile u / (g + 1), head slot u % (g + 1)

  if (threadIdx.x == 0) {
    bwd_init_bars(bars, bwd::EL_WARPS);
    tma_prefetch_desc(&mK);
    tma_prefetch_desc(&mV);
    tma_prefetch_desc(&mQ);
    tma_prefetch_desc(&mH);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0 && n_units > 0) {
      // ------------------------------------------------------------ TMA producer
      mbar_expect_tx(&bars->fixed_full, 5 * BOX_BIG);
      const int yk = int((long long)j * p.M + (long long)b * p.T + k0);
#pragma unroll
      for (int c = 0; c < 3; ++c) tma_load_2d(smem + A_K_OFF + c * BOX_BIG, &mK, &bars->fixed_full, 64 * c, yk);
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tma_load_2d(smem + A_V_OFF + c * BOX_BIG, &mV, &bars->fixed_full, j * 256 + 128 + 64 * c, b * p.T + k0);
      uint32_t issued = 0, par = 0;
      for (int u = 0; u < n_units; ++u) {
        const int s = u % NST;
        const uint32_t ph = (u / NST) & 1;
        if (u >= NST && !mbar_wait(&bars->empty[s], ph ^ 1, ctl, SITE_BWD_PRODUCER)) break;
        const int h = head_of(u % (g + 1), j, p.n_signal, g);
        const int t0 = q_begin + (u / (g + 1)) * TQ;
        const int y = int((long long)h * p.M + (long long)b * p.T + t0);
        uint8_t* st = smem + A_RING + s * STAGE;
        mbar_expect_tx(&bars->full[s], STAGE);
#pragma unroll
        for (int c = 0; c < 3; ++c) tma_load_2d(st + c * BOX_SMALL, &mQ, &bars->full[s], 64 * c, y);
#pragma unroll
        for (int c = 0; c < 2; ++c) tma_load_2d(st + (3 + c) * BOX_SMALL, &mH, &bars->full[s], 64 * c, y);
        issued |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      }
      for (int s = 0; s < NST; ++s)
        if (issued & (1u << s)) mbar_drain(&bars->full[s], (par >> s) & 1, ctl.err);
      mbar_drain(&bars->fixed_full, 0, ctl.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_units > 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = make_idesc(128, TQ, 0, 0, 0);     // S^T, dP^T (fp16)
      constexpr uint32_t idesc_dv = make_idesc(128, 128, 0, 0, 1);   // dV: B = dH, MN-major
      constexpr uint32_t idesc_dk = make_idesc(128, 192, 0, 0, 1);   // dK: B = q, MN-major
      const uint32_t hi = uint32_t(sdesc_sw128(smem_u32(smem), 16, 1024) >> 32);
      const uint32_t k_lo = uint32_t(sdesc_sw128(smem_u32(smem + A_K_OFF), 16, 1024));
      const uint32_t v_lo = uint32_t(sdesc_sw128(smem_u32(smem + A_V_OFF), 16, 1024));
      const uint32_t r_lo = uint32_t(sdesc_sw128(smem_u32(smem + A_RING), 16, 1024));
      const uint32_t rmn_lo = uint32_t(sdesc_sw128(smem_u32(smem + A_RING), BOX_SMALL, 1024));
      // dV += P^T dH and dK += dS'^T q of unit v; then its stage is free.  Slot v % 3 holds, for
      // the queries QG e .. QG e + QG - 1 of group e, P^T in columns QG e .. QG e + QG / 2 - 1
      // and dS'^T in the next QG / 2 (fp16 pairs): K step kk starts at el_col(kk) (+ QG / 2)
      auto issue_dvdk = [&](int v) -> bool {
        if (!mbar_wait(&bars->p_ready, v & 1, ctl, SITE_BWD_MMA)) return false;
        tc_fence_after();
        const uint32_t slot = tmem + 64 * uint32_t(v % 3);
        const uint32_t stmn = rmn_lo + uint32_t((v % NST) * (STAGE / 16));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)       // K = 64 queries
          mma_ts_w(tmem + T_DV, slot + el_col(kk), stmn + uint32_t(3 * (BOX_SMALL / 16) + kk * 128), hi, idesc_dv,
                   (v > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_w(tmem + T_DK, slot + el_col(kk) + QG / 2, stmn + uint32_t(kk * 128), hi, idesc_dk,
                   (v > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[v % NST]);
        mma_commit(&bars->dvdk_done);
        return true;
      };
      bool ok = mbar_wait(&bars->fixed_full, 0, ctl, SITE_BWD_MMA);
      tc_fence_after();
      for (int u = 0; u < n_units && ok; ++u) {
        const int s = u % NST;
        if (!mbar_wait(&bars->full[s], (u / NST) & 1, ctl, SITE_BWD_MMA)) { ok = false; break; }
        // slot u % 3 held dP^T(u - 1) (read by now?) and slot (u + 1) % 3 held P^T | dS'^T of
        // unit u - 2 (consumed by its dV / dK?)
        if (u >= 1 && !mbar_wait(&bars->el_read, (u - 1) & 1, ctl, SITE_BWD_MMA)) { ok = false; break; }
        if (u >= 2 && !mbar_wait(&bars->dvdk_done, (u - 2) & 1, ctl, SITE_BWD_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = r_lo + uint32_t(s * (STAGE / 16));
        const uint32_t tS = tmem + 64 * uint32_t(u % 3), tD = tmem + 64 * uint32_t((u + 1) % 3);
#pragma unroll
        for (int kk = 0; kk < 12; ++kk)      // S^T = [K^C | k^R] [q^C | q^R]^T, K 192
          mma_ss_w(tS, k_lo + uint32_t((kk >> 2) * (BOX_BIG / 16) + (kk & 3) * 2), hi,
                   st + uint32_t((kk >> 2) * (BOX_SMALL / 16) + (kk & 3) * 2), hi, idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)       // dP^T = V dH^T, K 128
          mma_ss_w(tD, v_lo + uint32_t((kk >> 2) * (BOX_BIG / 16) + (kk & 3) * 2), hi,
                   st + uint32_t((3 + (kk >> 2)) * (BOX_SMALL / 16) + (kk & 3) * 2), hi, idesc_s, kk > 0);
        mma_commit(&bars->s_full);
        if (u >= 1 && !issue_dvdk(u - 1)) { ok = false; break; }
      }
      if (ok && !issue_dvdk(n_units - 1)) ok = false;
      if (ok) mma_commit(&bars->acc_done);
      mma_commit(&bars->mma_final);
      mbar_drain(&bars->mma_final, 0, ctl.err);
    }
  } else {
    // ------------------------------------------------------------ elementwise (warps 2 ..)
    const int q = warp & 3;
    const int hq = (warp - 2) >> 2;            // group: queries QG hq .. QG hq + QG - 1 of a unit
    const int r = 32 * q + lane;
    const int s_key = k0 + r;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    // per warp: -lse and -Delta / sqrt(192) of its 32 queries of the unit
    float* ld = reinterpret_cast<float*>(smem + A_LD_OFF) + (warp - 2) * 2 * QG;
    bool ok = n_units > 0;
    // -lse / -Delta of a unit's QG queries, lane i (and i + 32) holding entry i of the staging;
    // the next unit's are loaded while this one is processed
    constexpr int NPRE = 2 * QG / 32;
    auto fetch_ld = [&](int uu, float* pre) {
      const int hh = head_of(uu % (g + 1), j, p.n_signal, g);
      const long long o = ((long long)hh * p.B + b) * p.Tpad + q_begin + (uu / (g + 1)) * TQ + QG * hq;
#pragma unroll
      for (int e = 0; e < NPRE; ++e) {
        const int i = lane + 32 * e;
        pre[e] = i < QG ? -p.lseT[o + i] : -p.deltaT[o + i - QG] * p.scale;
      }
    };
    float pre[NPRE];
    if (n_units > 0) fetch_ld(0, pre);
    for (int u = 0; u < n_units && ok; ++u) {
      const int t0 = q_begin + (u / (g + 1)) * TQ;
      __syncwarp();
#pragma unroll
      for (int e = 0; e < NPRE; ++e) ld[lane + 32 * e] = pre[e];
      __syncwarp();
      if (u + 1 < n_units) fetch_ld(u + 1, pre);
      // every (query, key) pair of the unit visible: no per-element mask
      const bool interior = t0 >= k0 + BK - 1 && t0 + TQ <= p.T && k0 + BK <= p.T &&
                            (p.window <= 0 || t0 + TQ - 1 - k0 < p.window);
      const bool w = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, u & 1, ctl, SITE_BWD_SOFTMAX));
      if (!w) { ok = false; break; }
      tc_fence_after();
      // this group's QG columns of S^T and dP^T
      const uint32_t tS = tmem + 64 * uint32_t(u % 3) + QG * hq + lane_off;
      const uint32_t tD = tmem + 64 * uint32_t((u + 1) % 3) + QG * hq + lane_off;
      // dP^T first: once every warp has read it, its slot is free for the next unit's S^T (S^T's
      // own slot receives P^T | dS'^T, each group writing only the columns it has read)
      uint32_t dv[QG], sv[QG];
      el_tmem_ld(tD, dv);
      el_tmem_ld(tS, sv);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->el_read);
      uint32_t pk[QG / 2], gk[QG / 2];
#pragma unroll
      for (int k = 0; k < QG / 4; ++k) {            // 4 queries: -lse and -Delta / sqrt(192) from the staging
        const float4 l4 = *reinterpret_cast<const float4*>(ld + 4 * k);
        const float4 d4 = *reinterpret_cast<const float4*>(ld + QG + 4 * k);
        const float nl[4] = {l4.x, l4.y, l4.z, l4.w}, nd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 2 * k + e;             // pair index within the 32 queries
          float x0, x1, p0, p1, d0, d1, g0, g1;
          ffma2vv(x0, x1, __uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]), p.scale_log2, p.scale_log2,
                  nl[2 * e], nl[2 * e + 1]);
          if ((i & 3) == 3) {
            exp2_poly2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          if (!interior) {
            const int qi = QG * hq + 2 * i;
            p0 = bwd_visible(t0 + qi, s_key, p.T, p.window) ? p0 : 0.f;
            p1 = bwd_visible(t0 + qi + 1, s_key, p.T, p.window) ? p1 : 0.f;
          }
          pk[i] = pack_half2(p0, p1);
          // dS' = P (dP - Delta) / sqrt(192)
          ffma2vv(d0, d1, __uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1]), p.scale, p.scale,
                  nd[2 * e], nd[2 * e + 1]);
          fmul2v(g0, g1, p0, p1, d0, d1);
          gk[i] = pack_half2(g0, g1);
        }
      }
      el_tmem_st_half(tS, pk);                 // P^T, QG / 2 columns of fp16 pairs
      el_tmem_st_half(tS + QG / 2, gk);        // dS'^T
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready);
    }
    // ---- dV and dK of this CTA's keys: 128 dV columns, then 192 dK columns, five chunks of 32
    // per half
    if (ok) {
      const bool w = __all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, ctl, SITE_BWD_SOFTMAX));
      if (w) {
        tc_fence_after();
        const long long m = (long long)b * p.T + s_key;
        const bool row_ok = s_key < p.T;
#pragma unroll 1
        for (int c = hq; c < 10; c += EL_GROUPS) {
          uint32_t v[32];
          GDLA_TMEM_LD32(tmem + T_DV + 32 * c + lane_off, v);
          tmem_ld_wait();
          if (!row_ok) continue;
          float* dst = c < 4 ? p.d_kv + m * p.n_groups * 256 + j * 256 + 128 + 32 * c
                             : p.dK + (m * p.n_groups + j) * 192 + 32 * (c - 4);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                              __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
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

// =================================================================== queries stationary: dq
// Grid (head, query block from the last, sequence): the heaviest causal blocks launch first.
// Roles (THREADS threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2 .. 1 +
// EL_WARPS elementwise, EL_GROUPS threads per query.
__global__ void __launch_bounds__(bwd::THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mH,
                  const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                  const __grid_constant__ BwdTcParams p, KernelCtl ctl) {
  using namespace bwd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = bwd_align(smem_raw);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + B_BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, qb = int(gridDim.y) - 1 - int(blockIdx.y), b = blockIdx.z;
  const int g = p.n_signal / p.n_groups;
  const int nH = p.n_signal + p.n_groups;
  const int j = h < p.n_signal ? h / g : h - p.n_signal;
  const int q0 = qb * BQ;
  const int s_lo = p.window > 0 ? max(0, q0 - p.window + 1) : 0;
  const int s_hi = min(p.T, q0 + BQ);
  const int k_begin = (s_lo / TK) * TK;
  const int n_units = s_hi > k_begin ? (s_hi - k_begin + TK - 1) / TK : 0;

  if (threadIdx.x == 0) {
    bwd_init_bars(bars, bwd::EL_WARPS);
    tma_prefetch_desc(&mQ);
    tma_prefetch_desc(&mH);
    tma_prefetch_desc(&mK);
    tma_prefetch_desc(&mV);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0 && n_units > 0) {
      // ------------------------------------------------------------ TMA producer
      mbar_expect_tx(&bars->fixed_full, 5 * BOX_BIG);
      const int yq = int((long long)h * p.M + (long long)b * p.T + q0);
#pragma unroll
      for (int c = 0; c < 3; ++c) tma_load_2d(smem + B_Q_OFF + c * BOX_BIG, &mQ, &bars->fixed_full, 64 * c, yq);
#pragma unroll
      for (int c = 0; c < 2; ++c) tma_load_2d(smem + B_H_OFF + c * BOX_BIG, &mH, &bars->fixed_full, 64 * c, yq);
      uint32_t issued = 0, par = 0;
      for (int u = 0; u < n_units; ++u) {
        const int s = u % NST;
        const uint32_t ph = (u / NST) & 1;
        if (u >= NST && !mbar_wait(&bars->empty[s], ph ^ 1, ctl, SITE_BWD_PRODUCER)) break;
        const int s0 = k_begin + u * TK;
        uint8_t* st = smem + B_RING + s * STAGE;
        mbar_expect_tx(&bars->full[s], STAGE);
        const int yk = int((long long)j * p.M + (long long)b * p.T + s0);
#pragma unroll
        for (int c = 0; c < 3; ++c) tma_load_2d(st + c * BOX_SMALL, &mK, &bars->full[s], 64 * c, yk);
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_2d(st + (3 + c) * BOX_SMALL, &mV, &bars->full[s], j * 256 + 128 + 64 * c, b * p.T + s0);
        issued |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      }
      for (int s = 0; s < NST; ++s)
        if (issued & (1u << s)) mbar_drain(&bars->full[s], (par >> s) & 1, ctl.err);
      mbar_drain(&bars->fixed_full, 0, ctl.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_units > 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = make_idesc(128, TK, 0, 0, 0);
      constexpr uint32_t idesc_dq = make_idesc(128, 192, 0, 0, 1);    // B = K tile, MN-major
      const uint32_t hi = uint32_t(sdesc_sw128(smem_u32(smem), 16, 1024) >> 32);
      const uint32_t q_lo = uint32_t(sdesc_sw128(smem_u32(smem + B_Q_OFF), 16, 1024));
      const uint32_t h_lo = uint32_t(sdesc_sw128(smem_u32(smem + B_H_OFF), 16, 1024));
      const uint32_t r_lo = uint32_t(sdesc_sw128(smem_u32(smem + B_RING), 16, 1024));
      const uint32_t rmn_lo = uint32_t(sdesc_sw128(smem_u32(smem + B_RING), BOX_SMALL, 1024));
      // dq += dS'(v) K(v) once the elementwise threads have written dS'(v); then the key tile's
      // stage and the S / dP buffer of v are free.  dS' of the keys QG e .. QG e + QG - 1 of group
      // e is in dP columns QG e .. QG e + QG / 2 - 1 (fp16 pairs): K step kk starts at el_col(kk)
      auto issue_dq = [&](int v) -> bool {
        const int buf = v & 1;
        if (!mbar_wait(&bars->p_ready2[buf], (v >> 1) & 1, ctl, SITE_BWD_MMA)) return false;
        tc_fence_after();
        const uint32_t stmn = rmn_lo + uint32_t((v % NST) * (STAGE / 16));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)       // dq += dS' [K^C | k^R], K = 64 keys
          mma_ts_w(tmem + T_DQ, tmem + T_DP + 128 * buf + el_col(kk), stmn + uint32_t(kk * 128), hi, idesc_dq,
                   (v > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[v % NST]);
        mma_commit(&bars->buf_free2[buf]);
        return true;
      };
      bool ok = mbar_wait(&bars->fixed_full, 0, ctl, SITE_BWD_MMA);
      tc_fence_after();
      for (int u = 0; u < n_units && ok; ++u) {
        const int s = u % NST, buf = u & 1;
        if (!mbar_wait(&bars->full[s], (u / NST) & 1, ctl, SITE_BWD_MMA)) { ok = false; break; }
        // dq(u - 2) must have read the dS' of this buffer
        if (u >= 2 && !mbar_wait(&bars->buf_free2[buf], ((u - 2) >> 1) & 1, ctl, SITE_BWD_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = r_lo + uint32_t(s * (STAGE / 16));
#pragma unroll
        for (int kk = 0; kk < 12; ++kk)      // S = [q^C | q^R] [K^C | k^R]^T
          mma_ss_w(tmem + T_S + 128 * buf, q_lo + uint32_t((kk >> 2) * (BOX_BIG / 16) + (kk & 3) * 2), hi,
                   st + uint32_t((kk >> 2) * (BOX_SMALL / 16) + (kk & 3) * 2), hi, idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)       // dP = dH V^T
          mma_ss_w(tmem + T_DP + 128 * buf, h_lo + uint32_t((kk >> 2) * (BOX_BIG / 16) + (kk & 3) * 2), hi,
                   st + uint32_t((3 + (kk >> 2)) * (BOX_SMALL / 16) + (kk & 3) * 2), hi, idesc_s, kk > 0);
        mma_commit(&bars->s_full2[buf]);
        if (u >= 1 && !issue_dq(u - 1)) { ok = false; break; }
      }
      if (ok && !issue_dq(n_units - 1)) ok = false;
      if (ok) mma_commit(&bars->acc_done);
      mma_commit(&bars->mma_final);
      mbar_drain(&bars->mma_final, 0, ctl.err);
    }
  } else {
    // ------------------------------------------------------------ elementwise (warps 2 ..)
    // EL_GROUPS threads per query: group e takes the keys QG e .. QG e + QG - 1 of a tile
    const int q = warp & 3;
    const int hk = (warp - 2) >> 2;
    const int r = 32 * q + lane;
    const int t = q0 + r;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const long long lo = ((long long)h * p.B + b) * p.Tpad + t;
    const float nl = t < p.T ? -p.lseT[lo] : 0.f;                 // -lse
    const float nd = t < p.T ? -p.deltaT[lo] * p.scale : 0.f;     // -Delta / sqrt(192)
    bool ok = n_units > 0;
    for (int u = 0; u < n_units && ok; ++u) {
      const int s0 = k_begin + u * TK, buf = u & 1;
      // every (query, key) pair of the tile visible: no per-element mask
      const bool interior = s0 + TK - 1 <= q0 && q0 + BQ <= p.T && (p.window <= 0 || q0 + BQ - 1 - s0 < p.window);
      const bool w = __all_sync(0xffffffffu, mbar_wait(&bars->s_full2[buf], (u >> 1) & 1, ctl, SITE_BWD_SOFTMAX));
      if (!w) { ok = false; break; }
      tc_fence_after();
      // this group's QG columns of S and dP; dS' (fp16 pairs) goes over the first QG / 2 of those
      // dP columns, which only this group reads
      const uint32_t tS = tmem + T_S + 128 * buf + QG * hk + lane_off;
      const uint32_t tD = tmem + T_DP + 128 * buf + QG * hk + lane_off;
      uint32_t sv[QG], dv[QG];
      el_tmem_ld(tS, sv);
      el_tmem_ld(tD, dv);
      tmem_ld_wait();
      uint32_t gk[QG / 2];
#pragma unroll
      for (int i = 0; i < QG / 2; ++i) {
        float x0, x1, p0, p1, d0, d1, g0, g1;
        ffma2(x0, x1, __uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]), p.scale_log2, nl);
        if ((i & 3) == 3) {
          exp2_poly2(x0, x1, p0, p1);
        } else {
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        if (!interior) {
          const int ks = s0 + QG * hk + 2 * i;
          p0 = bwd_visible(t, ks, p.T, p.window) ? p0 : 0.f;
          p1 = bwd_visible(t, ks + 1, p.T, p.window) ? p1 : 0.f;
        }
        ffma2(d0, d1, __uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1]), p.scale, nd);
        fmul2v(g0, g1, p0, p1, d0, d1);
        gk[i] = pack_half2(g0, g1);
      }
      el_tmem_st_half(tD, gk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready2[buf]);
    }
    if (ok) {
      const bool w = __all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, ctl, SITE_BWD_SOFTMAX));
      if (w) {
        tc_fence_after();
        const long long m = (long long)b * p.T + t;
#pragma unroll 1
        for (int c = hk; c < 6; c += EL_GROUPS) {   // dq^C (128 columns), then dq^R (64)
          uint32_t v[32];
          GDLA_TMEM_LD32(tmem + T_DQ + 32 * c + lane_off, v);
          tmem_ld_wait();
          if (t >= p.T) continue;
          float* dst = p.d_qq + m * nH * 192 +
                       (c < 4 ? (long long)h * 128 + 32 * c : (long long)nH * 128 + (long long)h * 64 + 32 * (c - 4));
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                              __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
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

// =================================================================== elementwise kernels
// ---- per (row m, KV group j): dDg -> dH of the group's four signal heads and its noise head
// (fp16, head-major rows for the tensor-core kernels), Delta of all five and the transposed
// log-sum-exp (head-major, sequences padded to Tpad rows), dlambda, dG.  One warp; lane owns
// columns 4 lane .. 4 lane + 3.
__global__ void bwd_pre_kernel(const __nv_bfloat16* __restrict__ dDg, const __nv_bfloat16* __restrict__ G,
                               const float* __restrict__ lam, const __nv_bfloat16* __restrict__ H,
                               const float* __restrict__ lse, long long M, int T, int B, int Tpad, int n_groups,
                               int n_signal, __half* __restrict__ dOT, float* __restrict__ deltaT,
                               float* __restrict__ lseT, float* __restrict__ dlam, float* __restrict__ dG) {
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= M * n_groups) return;
  const long long m = wid / n_groups;
  const int j = int(wid % n_groups);
  const int nH = n_signal + n_groups;
  const int g = n_signal / n_groups;
  const int c0 = 4 * lane;
  const long long tp = (m / T) * Tpad + m % T;      // padded row of m within its head
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
      dOT[((long long)s * M + m) * 128 + c0 + e] = __float2half_rn(dh[e]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      acc_delta += __shfl_xor_sync(0xffffffffu, acc_delta, o);
      acc_dl += __shfl_xor_sync(0xffffffffu, acc_dl, o);
    }
    if (lane == 0) {
      deltaT[(long long)s * B * Tpad + tp] = acc_delta;
      lseT[(long long)s * B * Tpad + tp] = lse[m * nH + s];
      dlam[row] = acc_dl;
    }
  }
  float acc = 0.f;
  const int hn_id = n_signal + j;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    dOT[((long long)hn_id * M + m) * 128 + c0 + e] = __float2half_rn(dhn[e]);
    acc += dhn[e] * hn[e];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    deltaT[(long long)hn_id * B * Tpad + tp] = acc;
    lseT[(long long)hn_id * B * Tpad + tp] = lse[m * nH + hn_id];
  }
}

// q rows of every head as [q^C | rotated q^R] (192 halves), head-major: Q192T[h][m] from the QQ
// row layout (q^C of all heads, then q^R of all heads).  One thread per 16-byte chunk.
__global__ void bwd_gather_q_kernel(const __half* __restrict__ QQ, long long M, int nH, __half* __restrict__ Q192T) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= M * nH * 24) return;
  const int ch = int(t % 24);
  const long long mh = t / 24;
  const long long m = mh / nH;
  const int h = int(mh % nH);
  const __half* src = ch < 16 ? QQ + m * nH * 192 + (long long)h * 128 + ch * 8
                              : QQ + m * nH * 192 + (long long)nH * 128 + (long long)h * 64 + (ch - 16) * 8;
  *reinterpret_cast<uint4*>(Q192T + ((long long)h * M + m) * 192 + ch * 8) = *reinterpret_cast<const uint4*>(src);
}

// key rows of every KV group as [K^C_j | rotated k^R] (192 halves), group-major: K192T[j][m].
__global__ void bwd_gather_k_kernel(const __half* __restrict__ KV, const __half* __restrict__ kR, long long M,
                                    int n_groups, __half* __restrict__ K192T) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= M * n_groups * 24) return;
  const int ch = int(t % 24);
  const long long mj = t / 24;
  const long long m = mj / n_groups;
  const int j = int(mj % n_groups);
  const __half* src = ch < 16 ? KV + m * n_groups * 256 + (long long)j * 256 + ch * 8 : kR + m * 64 + (ch - 16) * 8;
  *reinterpret_cast<uint4*>(K192T + ((long long)j * M + m) * 192 + ch * 8) = *reinterpret_cast<const uint4*>(src);
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

// =================================================================== host side
static int bwd_tpad(int T) { return (T + 63) / 64 * 64; }

size_t attn_bwd_workspace_bytes(long long M, int T, int n_heads, int n_groups) {
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  const long long B = M / T;
  const size_t padded = (size_t)n_heads * B * bwd_tpad(T) + 64;
  return al(M * n_heads * 128 * 2) + 2 * al(padded * 4) + al(M * n_heads * 192 * 2) +
         al(M * n_groups * 192 * 2) + al(M * n_groups * 192 * 4);
}

int launch_attn_bwd(const AttnBwdParams& a, const KernelCtlHost& ctlh, cudaStream_t st) {
  const long long M = (long long)a.B * a.T;
  const int nH = a.n_signal + a.n_groups, ng = a.n_groups;
  const int Tpad = bwd_tpad(a.T);
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  const size_t padded = (size_t)nH * a.B * Tpad + 64;
  uint8_t* w = static_cast<uint8_t*>(a.ws);
  __half* dOT = reinterpret_cast<__half*>(w); w += al(M * nH * 128 * 2);
  float* deltaT = reinterpret_cast<float*>(w); w += al(padded * 4);
  float* lseT = reinterpret_cast<float*>(w); w += al(padded * 4);
  __half* Q192T = reinterpret_cast<__half*>(w); w += al(M * nH * 192 * 2);
  __half* K192T = reinterpret_cast<__half*>(w); w += al(M * ng * 192 * 2);
  float* dK192 = reinterpret_cast<float*>(w);

  const __half* QQ = static_cast<const __half*>(a.QQ);
  const __half* KV = static_cast<const __half*>(a.KV);
  const __half* KR = static_cast<const __half*>(a.kR16);
  {
    const long long warps = M * ng;
    bwd_pre_kernel<<<unsigned((warps + 7) / 8), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.d_dg), static_cast<const __nv_bfloat16*>(a.G), a.lam,
        static_cast<const __nv_bfloat16*>(a.H), a.lse, M, a.T, a.B, Tpad, ng, a.n_signal, dOT, deltaT, lseT,
        a.d_lam, a.d_G);
    const long long nq_ch = M * nH * 24, nk_ch = M * ng * 24;
    bwd_gather_q_kernel<<<unsigned((nq_ch + 255) / 256), 256, 0, st>>>(QQ, M, nH, Q192T);
    bwd_gather_k_kernel<<<unsigned((nk_ch + 255) / 256), 256, 0, st>>>(KV, KR, M, ng, K192T);
    if (cudaPeekAtLastError() != cudaSuccess) return -4;
  }
  CUtensorMap mQ64, mQ128, mH64, mH128, mK64, mK128, mV64, mV128;
  const uint64_t qrows = (uint64_t)nH * M, krows = (uint64_t)ng * M;
  if (make_tmap_2d(&mQ64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q192T, 192, qrows, 384, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mQ128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Q192T, 192, qrows, 384, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mH64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, dOT, 128, qrows, 256, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mH128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, dOT, 128, qrows, 256, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mK64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, K192T, 192, krows, 384, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mK128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, K192T, 192, krows, 384, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mV64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, KV, (uint64_t)ng * 256, (uint64_t)M, (uint64_t)ng * 512, 64,
                   64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mV128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, KV, (uint64_t)ng * 256, (uint64_t)M, (uint64_t)ng * 512, 64,
                   128, CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  BwdTcParams p{};
  p.B = a.B; p.T = a.T; p.window = a.window; p.n_signal = a.n_signal; p.n_groups = ng; p.Tpad = Tpad; p.M = M;
  p.scale_log2 = a.scale_log2; p.scale = a.scale; p.lseT = lseT; p.deltaT = deltaT;
  p.dK = dK192; p.d_kv = a.d_kv; p.d_qq = a.d_qq;
  KernelCtl kc{ctlh.err, ctlh.limit_ns};
  if (cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd::A_SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd::B_SMEM) != cudaSuccess)
    return -4;
  bwd_dkdv_kernel<<<dim3(ng, (a.T + bwd::BK - 1) / bwd::BK, a.B), bwd::THREADS, bwd::A_SMEM, st>>>(mK128, mV128, mQ64, mH64,
                                                                                           p, kc);
  if (cudaPeekAtLastError() != cudaSuccess) return -4;
  bwd_dq_kernel<<<dim3(nH, (a.T + bwd::BQ - 1) / bwd::BQ, a.B), bwd::THREADS, bwd::B_SMEM, st>>>(mQ128, mH128, mK64, mV64, p,
                                                                                        kc);
  if (cudaPeekAtLastError() != cudaSuccess) return -4;
  const long long n_fin = M * ((long long)ng * 32 + 16);
  bwd_finish_k_kernel<<<unsigned((n_fin + 255) / 256), 256, 0, st>>>(dK192, M, ng, a.d_kv, a.d_kr);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
