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
// Work unit (one CTA): sequence b, KV head j, and 256 consecutive query positions split into
// two 128-row tiles ("slots").  The unit runs five passes, one per head of the group: first
// the noise head (its normalised output is parked in an fp32 scratch row per token), then the
// four signal heads, whose epilogue subtracts lambda times that row and applies the gate.
// Every pass streams the group's K/V tiles (128 keys) through an 8-deep ring of 16 KB TMA
// boxes (K^C low, K^C high, k^R; V low, V high) -- the tiles are shared by both slots, and the
// 16 KB k^R box is the single rotary key shared by all KV heads.
//
// Roles (384 threads):
//   warp 0      TMA producer (Q tiles per pass; K/V ring)
//   warp 1      TMEM owner; lane 0 issues tcgen05.mma:
//                 S_slot = Q_slot K^T   (M 128, N 128 keys, K 192; fp16 operands, fp32 in TMEM)
//                 O_slot += P_slot V    (P read from TMEM, two N = 64 halves of d_v)
//   warps 4-7   softmax / epilogue of slot 0 (thread = query row = TMEM lane)
//   warps 8-11  softmax / epilogue of slot 1
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512); P overwrites the first 64
// columns of S as packed fp16 pairs.  The MMA order PV0(i), QK0(i+1), PV1(i), QK1(i+1) keeps the
// tensor core busy with one slot while the other slot's softmax runs.  The running max is
// only moved (and O rescaled) when it grows by more than 2^8, which is exact after the final
// division by the row sum.
#include "gdla_common.cuh"
#include "gdla_internal.h"

namespace gdla {

namespace attn {
constexpr int RING = 8;
constexpr int SUB = 16384;                  // one 128 x 64 fp16 box
constexpr int Q_BYTES = 2 * 3 * SUB;        // 2 slots x (q^C lo, q^C hi, q^R)
constexpr int RING_OFF = Q_BYTES;
constexpr int BAR_OFF = RING_OFF + RING * SUB;
constexpr int SMEM = BAR_OFF + 256 + 1024;  // + barriers + alignment slack
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units
}  // namespace attn

struct AttnBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t ring_full[attn::RING], ring_empty[attn::RING];
  uint64_t s_full[2], p_ready[2], o_done[2], o_free[2];
  uint64_t mma_final;
  uint32_t tmem_base;
};

__device__ __forceinline__ uint8_t* attn_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__global__ void __launch_bounds__(384, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap mapQ,
                        const __grid_constant__ CUtensorMap mapKV,
                        const __grid_constant__ CUtensorMap mapKR,
                        const __grid_constant__ AttnParams p, KernelCtl ctl) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = attn_align(smem_raw);
  AttnBars* bars = reinterpret_cast<AttnBars*>(smem + BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: (sequence rows [rowbase, rowbase + T), KV head j, 256-row pair c), heaviest
  // causal units first.  Equal-length batches derive it from blockIdx; packed documents read
  // it from a schedule built on the device (surplus CTAs of the upper-bound grid exit here).
  int c, rowbase, T, j;
  if (p.units) {
    const int u = int(blockIdx.x) / p.n_groups;
    if (u >= *p.n_units) return;
    const int4 un = p.units[u];
    rowbase = un.x;
    T = un.y;
    c = un.z;
    j = int(blockIdx.x) % p.n_groups;
  } else {
    const int n_pairs = (p.T + 255) / 256;
    const int per_c = p.B * p.n_groups;
    c = n_pairs - 1 - int(blockIdx.x) / per_c;
    const int b = (int(blockIdx.x) % per_c) / p.n_groups;
    j = int(blockIdx.x) % p.n_groups;
    rowbase = b * p.T;
    T = p.T;
  }
  const int q0 = 256 * c;
  const int t_hi = min(T - 1, q0 + 255) / 128;
  const int t_lo = p.window > 0 ? max(0, q0 - p.window + 1) / 128 : 0;
  const int n_kv = t_hi - t_lo + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_ready[s], 128);
      mbar_init(&bars->o_done[s], 1);
      mbar_init(&bars->o_free[s], 128);
    }
    for (int s = 0; s < RING; ++s) {
      mbar_init(&bars->ring_full[s], 1);
      mbar_init(&bars->ring_empty[s], 1);
    }
    mbar_init(&bars->mma_final, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapKV);
    tma_prefetch_desc(&mapKR);
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
    if (lane == 0) {
      // ================================================================ TMA producer
      uint32_t ring_issued = 0, ring_par = 0, q_issued = 0, q_par = 0;
      uint32_t g = 0;
      bool ok = true;
      for (int pass = 0; pass < 5 && ok; ++pass) {
        const int h = pass == 0 ? p.n_signal + j : 4 * j + pass - 1;
        for (int s = 0; s < 2 && ok; ++s) {
          if (pass > 0 && !mbar_wait(&bars->q_empty[s], (pass - 1) & 1, ctl, SITE_ATTN_PRODUCER)) {
            ok = false;
            break;
          }
          uint8_t* qd = smem + s * 3 * SUB;
          const int y = rowbase + q0 + 128 * s;
          mbar_expect_tx(&bars->q_full[s], 3 * SUB);
          tma_load_2d(qd, &mapQ, &bars->q_full[s], h * 128, y);
          tma_load_2d(qd + SUB, &mapQ, &bars->q_full[s], h * 128 + 64, y);
          tma_load_2d(qd + 2 * SUB, &mapQ, &bars->q_full[s], p.rope_col0 + h * 64, y);
          q_issued |= 1u << s;
          q_par = (q_par & ~(1u << s)) | (uint32_t(pass & 1) << s);
        }
        for (int i = 0; i < n_kv && ok; ++i) {
          const int y = rowbase + 128 * (t_lo + i);
          for (int sub = 0; sub < 5; ++sub, ++g) {
            const int slot = g % RING;
            const uint32_t ph = (g / RING) & 1;
            if (g >= RING && !mbar_wait(&bars->ring_empty[slot], ph ^ 1, ctl, SITE_ATTN_PRODUCER)) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + RING_OFF + slot * SUB;
            mbar_expect_tx(&bars->ring_full[slot], SUB);
            if (sub == 2)
              tma_load_2d(dst, &mapKR, &bars->ring_full[slot], 0, y);
            else  // sub 0,1: K^C halves; 3,4: V halves
              tma_load_2d(dst, &mapKV, &bars->ring_full[slot], j * 256 + (sub < 2 ? sub : sub - 1) * 64, y);
            ring_issued |= 1u << slot;
            ring_par = (ring_par & ~(1u << slot)) | (ph << slot);
          }
        }
      }
      for (int s = 0; s < RING; ++s)
        if (ring_issued & (1u << s)) mbar_drain(&bars->ring_full[s], (ring_par >> s) & 1, ctl.err);
      for (int s = 0; s < 2; ++s)
        if (q_issued & (1u << s)) mbar_drain(&bars->q_full[s], (q_par >> s) & 1, ctl.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================================================================ MMA issuer
      constexpr uint32_t idesc_qk = make_idesc(128, 128, 0, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc(128, 64, 0, 0, 1);
      const uint32_t q_addr = smem_u32(smem);
      const uint32_t ring_addr = smem_u32(smem + RING_OFF);
      uint32_t g = 0, pr_par[2] = {0, 0};
      bool ok = true;

      auto wait_ring = [&](uint32_t gg, int n) -> bool {
        for (int k = 0; k < n; ++k) {
          const uint32_t idx = gg + k;
          if (!mbar_wait(&bars->ring_full[idx % RING], (idx / RING) & 1, ctl, SITE_ATTN_MMA))
            return false;
        }
        return true;
      };
      auto issue_qk = [&](int s, uint32_t gk) {
        const uint32_t d = tmem + s * 128;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int sub = kk >> 2, k4 = kk & 3;
          const uint64_t ad = sdesc_sw128(q_addr + (s * 3 + sub) * SUB + k4 * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(ring_addr + ((gk + sub) % RING) * SUB + k4 * 32, 16, 1024);
          mma_ss(d, ad, bd, idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int s, uint32_t gv, bool acc) {
        const uint32_t a = tmem + s * 128;
        const uint32_t d = tmem + 256 + s * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint64_t bd = sdesc_sw128(ring_addr + ((gv + hf) % RING) * SUB + kk * 2048, 8192, 1024);
            mma_ts(d + hf * 64, a + kk * 8, bd, idesc_pv, (acc || kk > 0) ? 1u : 0u);
          }
        }
      };
      auto release = [&](uint32_t gg, int n) {
        for (int k = 0; k < n; ++k) mma_commit(&bars->ring_empty[(gg + k) % RING]);
      };

      for (int pass = 0; pass < 5 && ok; ++pass) {
        if (!mbar_wait(&bars->q_full[0], pass & 1, ctl, SITE_ATTN_MMA) ||
            !mbar_wait(&bars->q_full[1], pass & 1, ctl, SITE_ATTN_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // prologue: S = Q K(0)^T for both slots
        uint32_t gk = g;
        if (!wait_ring(gk, 3)) { ok = false; break; }
        tc_fence_after();
        issue_qk(0, gk);
        mma_commit(&bars->s_full[0]);
        issue_qk(1, gk);
        mma_commit(&bars->s_full[1]);
        release(gk, 3);
        if (n_kv == 1) {
          mma_commit(&bars->q_empty[0]);
          mma_commit(&bars->q_empty[1]);
        }
        g += 3;
        for (int i = 0; i < n_kv; ++i) {
          const uint32_t gv = g;
          if (!wait_ring(gv, 2)) { ok = false; break; }
          g += 2;
          // ---- slot 0: O0 += P0 V
          if (i == 0 && pass > 0 && !mbar_wait(&bars->o_free[0], (pass - 1) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
          if (!mbar_wait(&bars->p_ready[0], pr_par[0], ctl, SITE_ATTN_MMA)) { ok = false; break; }
          pr_par[0] ^= 1;
          tc_fence_after();
          issue_pv(0, gv, i > 0);
          if (i == n_kv - 1) mma_commit(&bars->o_done[0]);
          // ---- slot 0: next S
          const bool more = i + 1 < n_kv;
          if (more) {
            gk = g;
            if (!wait_ring(gk, 3)) { ok = false; break; }
            tc_fence_after();
            issue_qk(0, gk);
            mma_commit(&bars->s_full[0]);
          }
          // ---- slot 1: O1 += P1 V
          if (i == 0 && pass > 0 && !mbar_wait(&bars->o_free[1], (pass - 1) & 1, ctl, SITE_ATTN_MMA)) { ok = false; break; }
          if (!mbar_wait(&bars->p_ready[1], pr_par[1], ctl, SITE_ATTN_MMA)) { ok = false; break; }
          pr_par[1] ^= 1;
          tc_fence_after();
          issue_pv(1, gv, i > 0);
          if (i == n_kv - 1) mma_commit(&bars->o_done[1]);
          release(gv, 2);
          if (more) {
            issue_qk(1, gk);
            mma_commit(&bars->s_full[1]);
            release(gk, 3);
            if (i + 1 == n_kv - 1) {
              mma_commit(&bars->q_empty[0]);
              mma_commit(&bars->q_empty[1]);
            }
            g += 3;
          }
        }
      }
      // every issued MMA must finish before TMEM is released
      mma_commit(&bars->mma_final);
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
    const int qpos = q0 + 128 * s + r;
    const bool row_valid = qpos < T;
    const long long m_row = (long long)rowbase + qpos;
    const int W = p.window;
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
        float mx = sc[0];
#pragma unroll
        for (int e = 1; e < 128; ++e) mx = fmaxf(mx, sc[e]);
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
        uint32_t pk[64];
        float lsum = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float p0 = ex2_approx(fmaf(sc[2 * e], p.scale_log2, neg_m));
          const float p1 = ex2_approx(fmaf(sc[2 * e + 1], p.scale_log2, neg_m));
          lsum += p0 + p1;
          pk[e] = pack_half2(p0, p1);
        }
        l_run += lsum;
        GDLA_TMEM_ST32(tS + 0, pk);
        GDLA_TMEM_ST32(tS + 32, (pk + 32));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_ready[s]);
      }
      if (!ok) break;

      // ---------------- epilogue of this pass
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
      mbar_arrive(&bars->o_free[s]);
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      if (!row_valid || m_row >= (long long)p.B * p.T || *reinterpret_cast<volatile int*>(ctl.err) != 0)
        continue;
      float* on_row = p.O_noise + (m_row * p.n_groups + j) * 128;
      if (pass == 0) {
#pragma unroll
        for (int e = 0; e < 128; e += 4)
          *reinterpret_cast<float4*>(on_row + e) =
              make_float4(__uint_as_float(ou[e]) * inv_l, __uint_as_float(ou[e + 1]) * inv_l,
                          __uint_as_float(ou[e + 2]) * inv_l, __uint_as_float(ou[e + 3]) * inv_l);
      } else {
        const int sig = 4 * j + pass - 1;
        const float lam = p.lam[m_row * p.n_signal + sig];
        const __nv_bfloat16* g_row =
            static_cast<const __nv_bfloat16*>(p.G) + (m_row * p.n_signal + sig) * 128;
        __nv_bfloat16* d_row = static_cast<__nv_bfloat16*>(p.Dg) + (m_row * p.n_signal + sig) * 128;
#pragma unroll
        for (int e = 0; e < 128; e += 8) {
          const uint4 gv = *reinterpret_cast<const uint4*>(g_row + e);
          const float4 n0 = *reinterpret_cast<const float4*>(on_row + e);
          const float4 n1 = *reinterpret_cast<const float4*>(on_row + e + 4);
          const float nn[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
          uint32_t outw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(&gw[q]);
            const float d0 = __uint_as_float(ou[e + 2 * q]) * inv_l - lam * nn[2 * q];
            const float d1 = __uint_as_float(ou[e + 2 * q + 1]) * inv_l - lam * nn[2 * q + 1];
            outw[q] = pack_bf162(sigmoidf_fast(__low2float(g2)) * d0,
                                 sigmoidf_fast(__high2float(g2)) * d1);
          }
          *reinterpret_cast<uint4*>(d_row + e) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
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

int launch_attn_prefill(const void* QQ, int qq_ld, const void* KV, const void* kR16,
                        const AttnParams& p, KernelCtlHost ctl, cudaStream_t st) {
  if (p.B <= 0 || p.T <= 0) return 0;
  const long long M = (long long)p.B * p.T;   // rows of the (packed) token matrix
  CUtensorMap mq, mkv, mkr;
  if (make_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, QQ, qq_ld, M, (uint64_t)qq_ld * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mkv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, KV, (uint64_t)p.n_groups * 256, M,
                   (uint64_t)p.n_groups * 256 * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      make_tmap_2d(&mkr, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kR16, 64, M, 128, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  if (cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           attn::SMEM) != cudaSuccess)
    return -4;
  const int grid = p.units ? p.max_units * p.n_groups : ((p.T + 255) / 256) * p.B * p.n_groups;
  KernelCtl kc{ctl.err, ctl.limit_ns};
  attn_prefill_kernel<<<grid, 384, attn::SMEM, st>>>(mq, mkv, mkr, p, kc);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla
