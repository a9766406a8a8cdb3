// Fused GDLA prefill attention for sm_100a.
//
// What it computes (picx.dev "Motif 3" summary, section 2.2, grouped differential output and
// output gating; paperglide.net Figure 1 caption): for every query token t and KV head j,
// the noise head j and the g = 4 signal heads 4j..4j+3 each attend, under the causal or
// sliding-window mask, over keys k_s = [K^C_{j,s}; k^R_s] and values V_{j,s} of KV head j:
//   H_h = softmax_s(q_h . k_s / sqrt(192)) V
//   D_s = H_s - lambda_{t,s} H_noise(j)           Dg_s = sigmoid(G_{t,s}) (.) D_s
// and writes Dg (bf16, head-major) for the output projection.
//
// Work unit (one pair of CTAs on one TPC, a cluster of 2): sequence b, KV head j and 512
// consecutive query positions.  CTA rank r owns rows [256 r, 256 r + 256) of the block, split
// into two 128-row tiles ("slots").  The unit runs five passes, one per head of the group:
// first the noise head (its normalised output is parked in an fp32 scratch row per token),
// then the four signal heads, whose epilogue subtracts lambda times that row and applies the
// gate.  Every pass streams the group's keys in tiles of 128.
//
// The pair shares each tensor-core instruction (tcgen05 cta_group::2, M = 256): for
//   S_slot = Q_slot K^T   (M 256 = 2 x 128 rows, N 128 keys, K 192; fp16, fp32 in TMEM)
//   O_slot += P_slot V    (P read from TMEM, N = d_v 128)
// the A operand (Q or P) and the accumulator rows live in the CTA that owns the rows, while
// the B operand is split by columns: each CTA loads 64 of the tile's 128 keys of K^C / k^R
// and 64 of the 128 value columns of V.  A CTA therefore moves 40 KB per key tile (half of
// what a CTA computing the same 256 rows alone would load) and the freed shared memory holds
// three tiles of K and three of V in flight.
//
// Roles (384 threads per CTA):
//   warp 0      TMA producer, both CTAs (Q per pass; K and V rings).  Every load of the pair
//               completes on the leader's barrier, which the leader arms with both CTAs' bytes.
//   warp 1      TMEM owner in both CTAs; lane 0 of the leader (rank 0) issues the MMAs and
//               commits each completion to the barriers of both CTAs.
//   warps 4-7   softmax / epilogue of slot 0 (thread = query row = TMEM lane)
//   warps 8-11  softmax / epilogue of slot 1; each warp reports "P written" and "O read" to
//               the leader's barriers (8 warps per phase).
// TMEM columns per CTA: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P overwrites the
// first 64 columns of S as packed fp16 pairs.  The MMA order PV0(i), QK0(i+1), PV1(i),
// QK1(i+1) keeps the tensor core busy with one slot while the other slot's softmax runs.  The
// running max is only moved (and O rescaled) when it grows by more than 2^8, which is exact
// after the final division by the row sum.
#include "gdla_common.cuh"
#include "gdla_internal.h"

namespace gdla {


namespace attn {
constexpr int QSUB = 16384;                   // one 128-row x 64-column fp16 box
constexpr int KBOX = 8192;                    // 64 keys x 64 columns
constexpr int KSTAGE = 3 * KBOX;              // this CTA's K^C low, K^C high, k^R of one tile
constexpr int VSTAGE = 16384;                 // 128 keys x this CTA's 64 value columns
constexpr int KST = 3, VST = 3;               // tiles in flight
constexpr int Q_BYTES = 2 * 3 * QSUB;         // 2 slots x (q^C lo, q^C hi, q^R)
constexpr int K_OFF = Q_BYTES;
constexpr int V_OFF = K_OFF + KST * KSTAGE;
constexpr int BAR_OFF = V_OFF + VST * VSTAGE;
constexpr int SMEM = BAR_OFF + 256 + 1024;    // + barriers + alignment slack
constexpr float RESCALE_THRESHOLD = 8.0f;     // log2 units
constexpr uint16_t BOTH = 3;                  // commit to the barriers of both CTAs
}  // namespace attn

struct AttnBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[attn::KST], k_empty[attn::KST];
  uint64_t v_full[attn::VST], v_empty[attn::VST];
  uint64_t s_full[2], p_ready[2], o_done[2], o_free[2];
  uint64_t mma_final;
  uint32_t tmem_base;
};
static_assert(sizeof(AttnBars) <= 256, "barrier block");


// sigmoid(z) = 1 / (1 + 2^(-z log2 e)) with the approximate reciprocal-divide (2 ulp): the
// result is rounded to bf16.
__device__ __forceinline__ float sigmoid_approx(float z) {
  return __fdividef(1.0f, 1.0f + ex2_approx(-1.4426950408889634f * z));
}
__device__ __forceinline__ uint8_t* attn_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// SAVE: also write every head's normalised output and log-sum-exp (for the backward).
// PREFIX: keys and queries are different row ranges (a key prefix before the queries); without
// it the key rows are the query rows and the offsets fold away at compile time.
template <bool SAVE, bool PREFIX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap mapQ,
                        const __grid_constant__ CUtensorMap mapK,
                        const __grid_constant__ CUtensorMap mapKR,
                        const __grid_constant__ CUtensorMap mapV,
                        const __grid_constant__ AttnParams p, KernelCtl ctl) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = attn_align(smem_raw);
  AttnBars* bars = reinterpret_cast<AttnBars*>(smem + BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // the leader's copy of one of this CTA's barriers
  auto lead = [&](uint64_t* b) { return smem_map_rank(smem_u32(b), 0); };

  // ---- work unit: (query rows [rowbase, rowbase + T) of a sequence whose keys are the rows
  // [kvbase, kvbase + T_kv), KV head j, 512-row block c), heaviest causal units first.  Query
  // row t sits at key position q_off + t (q_off > 0: a key prefix precedes the queries).
  // Equal-length batches derive the unit from the pair index; packed documents read it from a
  // schedule built on the device (surplus pairs of the upper-bound grid exit here, both CTAs
  // of a pair together, before any cluster-wide step).
  const int pu = int(blockIdx.x) >> 1;
  int c, rowbase, kvbase, T, T_kv, q_off, j;
  if (p.units) {
    const int u = pu / p.n_groups;
    if (u >= *p.n_units) return;
    const int4 un = p.units[u];
    rowbase = kvbase = un.x;
    T = T_kv = un.y;
    q_off = 0;
    c = un.z;
    j = pu % p.n_groups;
  } else {
    const int n_blk = (p.T + 511) / 512;
    const int per_c = p.B * p.n_groups;
    c = n_blk - 1 - pu / per_c;
    const int b = (pu % per_c) / p.n_groups;
    j = pu % p.n_groups;
    rowbase = b * p.T;
    T = p.T;
    kvbase = PREFIX ? b * p.T_kv : rowbase;
    T_kv = PREFIX ? p.T_kv : T;
    q_off = PREFIX ? p.q_off : 0;
  }
  const int q0 = 512 * c;
  const int t_hi = min(T_kv - 1, q_off + q0 + 511) / 128;
  const int t_lo = p.window > 0 ? max(0, q_off + q0 - p.window + 1) / 128 : 0;
  const int n_kv = t_hi - t_lo + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_ready[s], 8);
      mbar_init(&bars->o_done[s], 1);
      mbar_init(&bars->o_free[s], 8);
    }
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->mma_final, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapKR);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars->tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before any cross-CTA arrive or copy
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ================================================================ TMA producer
      uint32_t kq = 0, vq = 0;
      uint32_t k_armed = 0, k_par = 0, v_armed = 0, v_par = 0, q_armed = 0, q_par = 0;
      bool ok = true;
      for (int pass = 0; pass < 5 && ok; ++pass) {
        const int h = pass == 0 ? p.n_signal + j : 4 * j + pass - 1;
        for (int s = 0; s < 2 && ok; ++s) {
          if (pass > 0 && !mbar_wait(&bars->q_empty[s], (pass - 1) & 1, ctl, SITE_ATTN_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* qd = smem + s * 3 * QSUB;
          const int y = rowbase + q0 + 256 * int(rank) + 128 * s;
          if (leader) {
            mbar_expect_tx(&bars->q_full[s], 2 * 3 * QSUB);
            q_armed |= 1u << s;
            q_par = (q_par & ~(1u << s)) | (uint32_t(pass & 1) << s);
          }
          const uint32_t bar = lead(&bars->q_full[s]);
          tma_load_2d_pair(qd, &mapQ, bar, h * 128, y);
          tma_load_2d_pair(qd + QSUB, &mapQ, bar, h * 128 + 64, y);
          tma_load_2d_pair(qd + 2 * QSUB, &mapQ, bar, p.rope_col0 + h * 64, y);
        }
        for (int i = 0; i < n_kv && ok; ++i) {
          const int y0 = kvbase + 128 * (t_lo + i);
          {  // this CTA's 64 keys of K^C and k^R
            const int st = kq % KST;
            const uint32_t ph = (kq / KST) & 1;
            if (kq >= KST && !mbar_wait(&bars->k_empty[st], ph ^ 1, ctl, SITE_ATTN_PRODUCER)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_expect_tx(&bars->k_full[st], 2 * KSTAGE);
              k_armed |= 1u << st;
              k_par = (k_par & ~(1u << st)) | (ph << st);
            }
            uint8_t* dst = smem + K_OFF + st * KSTAGE;
            const uint32_t bar = lead(&bars->k_full[st]);
            const int yk = y0 + 64 * int(rank);
            tma_load_2d_pair(dst, &mapK, bar, j * 256, yk);
            tma_load_2d_pair(dst + KBOX, &mapK, bar, j * 256 + 64, yk);
            tma_load_2d_pair(dst + 2 * KBOX, &mapKR, bar, 0, yk);
            ++kq;
          }
          {  // all 128 keys of this CTA's 64 value columns
            const int st = vq % VST;
            const uint32_t ph = (vq / VST) & 1;
            if (vq >= VST && !mbar_wait(&bars->v_empty[st], ph ^ 1, ctl, SITE_ATTN_PRODUCER)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_expect_tx(&bars->v_full[st], 2 * VSTAGE);
              v_armed |= 1u << st;
              v_par = (v_par & ~(1u << st)) | (ph << st);
            }
            tma_load_2d_pair(smem + V_OFF + st * VSTAGE, &mapV, lead(&bars->v_full[st]),
                             j * 256 + 128 + 64 * int(rank), y0);
            ++vq;
          }
        }
      }
      // the leader's barriers count both CTAs' copies: let every armed phase land
      for (int s = 0; s < KST; ++s)
        if (k_armed & (1u << s)) mbar_drain(&bars->k_full[s], (k_par >> s) & 1, ctl.err);
      for (int s = 0; s < VST; ++s)
        if (v_armed & (1u << s)) mbar_drain(&bars->v_full[s], (v_par >> s) & 1, ctl.err);
      for (int s = 0; s < 2; ++s)
        if (q_armed & (1u << s)) mbar_drain(&bars->q_full[s], (q_par >> s) & 1, ctl.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ================================================================ MMA issuer (leader)
      constexpr uint32_t idesc_qk = make_idesc(256, 128, 0, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc(256, 128, 0, 0, 1);
      const uint32_t q_addr = smem_u32(smem);
      const uint32_t k_addr = smem_u32(smem + K_OFF);
      const uint32_t v_addr = smem_u32(smem + V_OFF);
      uint32_t kq = 0, vq = 0, pr_par[2] = {0, 0};
      bool ok = true;

      // Descriptors are built once; an operand at byte offset o from a base adds o / 16 to the
      // low word (start-address field, 14 bits: no carry for offsets inside shared memory).
      const uint64_t dq = sdesc_sw128(q_addr, 16, 1024);
      const uint64_t dk = sdesc_sw128(k_addr, 16, 1024);
      const uint64_t dv = sdesc_sw128(v_addr, 8192, 1024);
      const uint32_t q_lo = uint32_t(dq), q_hi = uint32_t(dq >> 32);
      const uint32_t k_lo = uint32_t(dk), k_hi = uint32_t(dk >> 32);
      const uint32_t v_lo = uint32_t(dv), v_hi = uint32_t(dv >> 32);
      auto issue_qk = [&](int s, int kst) {
        const uint32_t d = tmem + s * 128;
        const uint32_t a0 = q_lo + uint32_t(s * 3 * QSUB >> 4);
        const uint32_t b0 = k_lo + uint32_t(kst * KSTAGE >> 4);
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int sub = kk >> 2, k4 = kk & 3;
          mma_ss_pair(d, a0 + uint32_t((sub * QSUB + k4 * 32) >> 4), q_hi,
                      b0 + uint32_t((sub * KBOX + k4 * 32) >> 4), k_hi, idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int s, int vst, bool acc) {
        const uint32_t a = tmem + s * 128;
        const uint32_t d = tmem + 256 + s * 128;
        const uint32_t b0 = v_lo + uint32_t(vst * VSTAGE >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_pair(d, a + kk * 8, b0 + uint32_t(kk * 2048 >> 4), v_hi, idesc_pv,
                      (acc || kk > 0) ? 1u : 0u);
      };

      for (int pass = 0; pass < 5 && ok; ++pass) {
        if (!mbar_wait(&bars->q_full[0], pass & 1, ctl, SITE_ATTN_MMA) ||
            !mbar_wait(&bars->q_full[1], pass & 1, ctl, SITE_ATTN_MMA)) {
          ok = false;
          break;
        }
        // prologue: S = Q K(0)^T for both slots
        int kst = kq % KST;
        if (!mbar_wait(&bars->k_full[kst], (kq / KST) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
        issue_qk(0, kst);
        mma_commit_pair(&bars->s_full[0], BOTH);
        issue_qk(1, kst);
        mma_commit_pair(&bars->s_full[1], BOTH);
        mma_commit_pair(&bars->k_empty[kst], BOTH);
        ++kq;
        if (n_kv == 1) {
          mma_commit_pair(&bars->q_empty[0], BOTH);
          mma_commit_pair(&bars->q_empty[1], BOTH);
        }
        for (int i = 0; i < n_kv; ++i) {
          const int vst = vq % VST;
          if (!mbar_wait(&bars->v_full[vst], (vq / VST) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
          // ---- slot 0: O0 += P0 V
          if (i == 0 && pass > 0 &&
              !mbar_wait(&bars->o_free[0], (pass - 1) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
          if (!mbar_wait(&bars->p_ready[0], pr_par[0], ctl, SITE_ATTN_MMA)) { ok = false; break; }
          pr_par[0] ^= 1;
          tc_fence_after();
          issue_pv(0, vst, i > 0);
          if (i == n_kv - 1) mma_commit_pair(&bars->o_done[0], BOTH);
          // ---- slot 0: next S
          const bool more = i + 1 < n_kv;
          if (more) {
            kst = kq % KST;
            if (!mbar_wait(&bars->k_full[kst], (kq / KST) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
            issue_qk(0, kst);
            mma_commit_pair(&bars->s_full[0], BOTH);
          }
          // ---- slot 1: O1 += P1 V
          if (i == 0 && pass > 0 &&
              !mbar_wait(&bars->o_free[1], (pass - 1) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
          if (!mbar_wait(&bars->p_ready[1], pr_par[1], ctl, SITE_ATTN_MMA)) { ok = false; break; }
          pr_par[1] ^= 1;
          tc_fence_after();
          issue_pv(1, vst, i > 0);
          if (i == n_kv - 1) mma_commit_pair(&bars->o_done[1], BOTH);
          mma_commit_pair(&bars->v_empty[vst], BOTH);
          ++vq;
          if (more) {
            issue_qk(1, kst);
            mma_commit_pair(&bars->s_full[1], BOTH);
            mma_commit_pair(&bars->k_empty[kst], BOTH);
            ++kq;
            if (i + 1 == n_kv - 1) {
              mma_commit_pair(&bars->q_empty[0], BOTH);
              mma_commit_pair(&bars->q_empty[1], BOTH);
            }
          }
        }
      }
      // every issued MMA (which reads the peer's shared memory and writes its TMEM) must
      // finish before either CTA passes the closing cluster barrier
      mma_commit_pair(&bars->mma_final, 1);
      mbar_drain(&bars->mma_final, 0, ctl.err);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax + epilogue
    const int s = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t tS = tmem + s * 128 + lane_off;
    const uint32_t tO = tmem + 256 + s * 128 + lane_off;
    const int qrow = q0 + 256 * int(rank) + 128 * s + r;   // query row within the sequence
    const int qpos = q_off + qrow;                           // its key position
    const bool row_valid = qrow < T;
    const long long m_row = (long long)rowbase + qrow;
    const int W = p.window;
    const uint32_t p_ready_cl = lead(&bars->p_ready[s]);
    const uint32_t o_free_cl = lead(&bars->o_free[s]);
    uint32_t sf_par = 0;
    bool ok = true;

    for (int pass = 0; pass < 5 && ok; ++pass) {
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = 0; i < n_kv; ++i) {
        bool w_ok = mbar_wait(&bars->s_full[s], sf_par, ctl, SITE_ATTN_SOFTMAX);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        sf_par ^= 1;
        tc_fence_after();
        uint32_t u[128];
        GDLA_TMEM_LD32(tS + 0, u);
        GDLA_TMEM_LD32(tS + 32, (u + 32));
        GDLA_TMEM_LD32(tS + 64, (u + 64));
        GDLA_TMEM_LD32(tS + 96, (u + 96));
        tmem_ld_wait();
        float sc[128];
#pragma unroll
        for (int e = 0; e < 128; ++e) sc[e] = __uint_as_float(u[e]);
        const int k0 = 128 * (t_lo + i);
        const bool need_mask = (k0 + 127 > qpos) || (W > 0 && k0 <= qpos - W);
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 128; ++e) {
            const int kp = k0 + e;
            if (kp > qpos || (W > 0 && kp <= qpos - W)) sc[e] = -INFINITY;
          }
        }
        // row max: eight independent chains of three-input maxima, then their maximum
        float cm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float m = fmax3f(sc[k], sc[k + 8], sc[k + 16]);
#pragma unroll
          for (int e = 24; e < 120; e += 16) m = fmax3f(m, sc[k + e], sc[k + e + 8]);
          cm[k] = fmaxf(m, sc[k + 120]);
        }
        const float mx = fmax3f(fmax3f(cm[0], cm[1], cm[2]), fmax3f(cm[3], cm[4], cm[5]), fmaxf(cm[6], cm[7]));
        const float m_tile = mx * p.scale_log2;
        float alpha = 1.f;
        bool resc = false;
        if (i == 0) {
          m_run = m_tile;
        } else if (m_tile > m_run + RESCALE_THRESHOLD) {
          alpha = ex2_approx(m_run - m_tile);
          m_run = m_tile;
          resc = true;
        }
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int cc = 0; cc < 128; cc += 32) {
            uint32_t o[32];
            GDLA_TMEM_LD32(tO + cc, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            GDLA_TMEM_ST32(tO + cc, o);
          }
          tmem_st_wait();
        }
        l_run *= alpha;
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
        // P = 2^(s * scale - m) as fp16 pairs over S's first 64 columns, written to TMEM in four
        // 32-key chunks; every fourth pair takes the FMA-pipe exponential
        float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int e = 16 * c + q;
            float x0, x1, p0, p1;
            ffma2(x0, x1, sc[2 * e], sc[2 * e + 1], p.scale_log2, neg_m);
            if ((e & 3) == 3) {
              exp2_poly2(x0, x1, p0, p1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            fadd2(ls[2 * (e & 3)], ls[2 * (e & 3) + 1], p0, p1);
            pk[q] = pack_half2(p0, p1);
          }
          GDLA_TMEM_ST16(tS + 16 * c, pk);
        }
        const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        l_run += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(p_ready_cl);
      }
      if (!ok) break;

      // ---------------- epilogue of this pass.  The parked noise rows are interleaved in
      // blocks of 32 rows (the rows of one warp), so a warp's accesses to them are contiguous;
      // the gate and noise operands are loaded a 32-column chunk at a time ahead of its math.
      bool w_ok = mbar_wait(&bars->o_done[s], pass & 1, ctl, SITE_ATTN_SOFTMAX);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) { ok = false; break; }
      tc_fence_after();
      uint32_t ou[128];
      GDLA_TMEM_LD32(tO + 0, ou);
      GDLA_TMEM_LD32(tO + 32, (ou + 32));
      GDLA_TMEM_LD32(tO + 64, (ou + 64));
      GDLA_TMEM_LD32(tO + 96, (ou + 96));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(o_free_cl);
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      if (!row_valid || m_row >= (long long)p.B * p.T || *reinterpret_cast<volatile int*>(ctl.err) != 0)
        continue;
      if (SAVE) {
        // for the backward: this head's normalised output and log2-sum-exp2 of its scores
        const int head = pass == 0 ? p.n_signal + j : 4 * j + pass - 1;
        const long long hrow = m_row * (p.n_signal + p.n_groups) + head;
        uint4* hd = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.H_out) + hrow * 128);
#pragma unroll
        for (int e = 0; e < 128; e += 8)
          hd[e / 8] = make_uint4(
              pack_bf162(__uint_as_float(ou[e]) * inv_l, __uint_as_float(ou[e + 1]) * inv_l),
              pack_bf162(__uint_as_float(ou[e + 2]) * inv_l, __uint_as_float(ou[e + 3]) * inv_l),
              pack_bf162(__uint_as_float(ou[e + 4]) * inv_l, __uint_as_float(ou[e + 5]) * inv_l),
              pack_bf162(__uint_as_float(ou[e + 6]) * inv_l, __uint_as_float(ou[e + 7]) * inv_l));
        p.lse_out[hrow] = m_run + __log2f(l_run);
      }
      // column quad e/4 of row m: ((m/32 * n_groups + j) * 32 + e/4) * 128 + (m%32) * 4
      float* on_q = p.O_noise + ((m_row >> 5) * p.n_groups + j) * 4096 + (m_row & 31) * 4;
      if (pass == 0) {
#pragma unroll
        for (int e = 0; e < 128; e += 4)
          *reinterpret_cast<float4*>(on_q + (e / 4) * 128) =
              make_float4(__uint_as_float(ou[e]) * inv_l, __uint_as_float(ou[e + 1]) * inv_l,
                          __uint_as_float(ou[e + 2]) * inv_l, __uint_as_float(ou[e + 3]) * inv_l);
      } else {
        const int sig = 4 * j + pass - 1;
        const float lam = p.lam[m_row * p.n_signal + sig];
        const uint4* g_row = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.G) + (m_row * p.n_signal + sig) * 128);
        uint4* d_row = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.Dg) + (m_row * p.n_signal + sig) * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 gv[4];
          float4 nv[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) gv[q] = __ldg(g_row + 4 * c + q);
#pragma unroll
          for (int q = 0; q < 8; ++q) nv[q] = *reinterpret_cast<const float4*>(on_q + (8 * c + q) * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float nn[8] = {nv[2 * q].x, nv[2 * q].y, nv[2 * q].z, nv[2 * q].w,
                                 nv[2 * q + 1].x, nv[2 * q + 1].y, nv[2 * q + 1].z, nv[2 * q + 1].w};
            const uint32_t gw[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
            const int e = 32 * c + 8 * q;
            uint32_t outw[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(&gw[h]);
              const float d0 = __uint_as_float(ou[e + 2 * h]) * inv_l - lam * nn[2 * h];
              const float d1 = __uint_as_float(ou[e + 2 * h + 1]) * inv_l - lam * nn[2 * h + 1];
              outw[h] = pack_bf162(sigmoid_approx(__low2float(g2)) * d0,
                                   sigmoid_approx(__high2float(g2)) * d1);
            }
            d_row[4 * c + q] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
          }
        }
      }
    }
  }

  // Neither CTA leaves (or frees TMEM) while the other may still touch its shared memory or
  // TMEM: the leader has waited for its last MMA, every role has returned from bounded waits.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

int launch_attn_prefill(const void* QQ, int qq_ld, const void* KV, const void* kR16,
                        const AttnParams& p, KernelCtlHost ctl, cudaStream_t st) {
  if (p.B <= 0 || p.T <= 0) return 0;
  if (p.T_kv < p.T + p.q_off || (p.units && (p.T_kv != p.T || p.q_off != 0))) return -2;
  const long long M = (long long)p.B * p.T;      // query rows of the (packed) token matrix
  const long long Mk = (long long)p.B * p.T_kv;  // key rows
  const uint64_t kv_ld = (uint64_t)p.n_groups * 256;
  CUtensorMap mq, mk, mkr, mv;
  if (make_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, QQ, qq_ld, M, (uint64_t)qq_ld * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, KV, kv_ld, Mk, kv_ld * 2, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mkr, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kR16, 64, Mk, 128, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, KV, kv_ld, Mk, kv_ld * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  const bool prefix = p.q_off != 0 || p.T_kv != p.T;
  if (p.H_out && (!p.lse_out || prefix)) return -2;
  auto kern = p.H_out ? attn_prefill_kernel<true, false>
                      : (prefix ? attn_prefill_kernel<false, true> : attn_prefill_kernel<false, false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, attn::SMEM) != cudaSuccess)
    return -4;
  const long long units = p.units ? (long long)p.max_units : (long long)((p.T + 511) / 512) * p.B;
  const long long grid = 2 * units * p.n_groups;   // two CTAs (one cluster) per unit
  if (grid > 0x7fffffffLL) return -2;
  KernelCtl kc{ctl.err, ctl.limit_ns};
  kern<<<unsigned(grid), 384, attn::SMEM, st>>>(mq, mk, mkr, mv, p, kc);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
