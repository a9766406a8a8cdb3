// Absorbed-form GDLA decode attention on the tensor cores (sm_100a), reading every cached byte
// into the SM once.
//
// For one query row r (one new token of one sequence) the 80 heads attend over the latent-cache
// rows c_p = [c_bar_p (512) | rotated k^R_p (64)] (the MLA weight absorption: q~_h =
// [W_UK q^C_h ; q^R_h], score_{h,p} = q~_h . c_p / sqrt(192); picx.dev Motif 3 summary, section
// 2.2, with K and V regrouped into the latent space).  Per 64-position tile:
//   S[h, p]    = q~[h, :] . C[p, :]        tcgen05.mma M 128 (heads, 80 used), N 64, K 576
//   P[h, p]    = 2^(S log2e / sqrt(192) - m_h)   (bf16, one thread per head, into shared memory)
//   O^T[l, h] += C[:, l]^T P[h, :]^T        4 x tcgen05.mma M 128 (latent rows), N 80, K 64
// The tile stays in shared memory from the score MMAs to the PV MMAs, so nothing is re-read.
// That needs room: q~ of 80 heads is 90 KB, so its first 256 latent dims live in TMEM as the
// A operand of the score MMA (128 columns), and only dims 256..575 (50 KB) in shared memory.
// TMEM: q~ part 128 columns | S 64 | O^T 4 x 80 = 512.  Shared memory: q~ part 50 KB, P 10 KB,
// a ring of nine 16 KB latent slots (two [64 positions][64 dims] boxes each) and two 8 KB
// rotary slots (a tile takes four latent slots and one rotary slot): about 2.2 tiles.
//
// Work split ("stream-K"): the key tiles of all rows form one list, the rows in token-major
// order (dec_list_pos: token 0 of every sequence, then token 1, ...); CTA c of G = min(grid, N)
// takes tiles [c N / G, (c + 1) N / G), i.e. one wave with equal work per SM whatever the cache
// lengths.  The piece of a row inside one CTA's range is a segment: it gets its own online
// softmax and writes a partial (m_h, l_h, O^T) to slot c + l (l: the row's list position); the
// merge kernel in decode.cu combines a row's segments.  With q_len new tokens per sequence the
// list is q_len nearly equal parts with the same tile positions, so CTAs c and c + G / q_len
// reach the same cache tiles at about the same time and the later reads hit L2.
//
// Roles (256 threads): warps 0-3 softmax and O^T epilogue (warp w reads TMEM lanes 32 w ..
// 32 w + 31: thread = head h = 32 w + lane for h < 80, thread = latent row for O^T), warp 4 TMA
// producer, warp 7 TMEM owner + score (S) MMA issuer, warp 6 PV MMA issuer, warp 5 idle (the
// MXFP8 form, 384 threads: warp 5 issues S, warp 11 PV, warps 6-9 convert).  Per tile J the
// tensor core runs S(J) as its units land and PV(J) once the softmax has written P(J): the two
// chains are issued by different threads, so the softmax of tile J overlaps PV(J - 1) and
// S(J + 1).  The single S buffer is released as soon as the softmax has read it into
// registers; the single P buffer is written once PV(J - 1) is done; the ring holds tiles J - 1
// and J plus one slot of J + 1.  The issuers step through precomputed descriptor words
// (rebuilding 64-bit descriptors per MMA had made the issue loop slower still).  A tile takes 36
// score MMAs of N 64 and 16 PV MMAs of N 80, about 75 cycles each to issue here; with one thread
// issuing all 52 that issue rate was the bound (traces showed the tile's units already landed
// when the issuer reached them), which is why the PV chain has its own thread.
// The running maximum m_h moves only when a score exceeds it by more than 2^8 (O^T and l_h are
// then rescaled), which is exact after the final division.  Rows of the last tile beyond the
// row's last key are zeroed in shared memory before the PV, so that a cache tail the caller
// never wrote (NaN, Inf) cannot reach the output through 0 * NaN.
//
// MXFP8 cache (template C8, rows of gdla_fp8.cuh): the producer loads a tile's rope codes and
// block scales first, then its latent codes into the upper half of each ring slot; four more
// warps (6-9, two threads per row) convert E4M3 x 2^k to fp16 in place, in the layout of the
// bf16 tiles, and zero the rows outside the key range; q~, P and the tiles are fp16 MMA
// operands.  The conversion adds to the per-tile chain above (slot freed -> codes loaded ->
// converted -> scores), so the half-size cache is not faster than the bf16 one.
#include "gdla_common.cuh"
#include "gdla_decode.h"
#include "gdla_fp8.cuh"
#include "gdla_internal.h"

namespace gdla {

namespace dsk {
constexpr int NH = 80;
constexpr int TP = 64;                          // positions per tile
constexpr int QS_BOX = NH * 128;                // [80 rows][64 bf16] box of q~ (10 KB)
constexpr int QS_OFF = 0;                       // q~ dims 256..575: 5 boxes
constexpr int P_OFF = QS_OFF + 5 * QS_BOX;      // P [80 heads][64 positions] bf16
constexpr int LAT_SLOT = 16384;                 // [64 pos][64 dims] x 2 (128 latent dims)
constexpr int NLAT = 9;
constexpr int ROPE_SLOT = 8192;                 // [64 pos][64 rope dims]
constexpr int NROPE = 2;
constexpr int LAT_OFF = P_OFF + NH * 128;
constexpr int ROPE_OFF = LAT_OFF + NLAT * LAT_SLOT;
constexpr int BAR_OFF = ROPE_OFF + NROPE * ROPE_SLOT;
constexpr int SMEM = BAR_OFF + 1024 + 1024;    // barriers + alignment slack
constexpr int QT_COL = 0, S_COL = 128, O_COL = 192;   // TMEM columns
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr int PREFETCH_AHEAD = 0;               // tiles of L2 prefetch ahead of the TMA loads (0: none;
                                                // measured no faster at 3, slower at 6 and 12)
static_assert(SMEM <= 232448, "shared memory");
// MXFP8 cache rows (608 bytes: 576 E4M3 codes, 18 block scales, padding): a tile's raw rows
// land by TMA in the upper half of each latent slot ([64 rows][128 codes], 8 KB) and after the
// first 2 KB of its rope slot ([64 rows][96 bytes]: 64 rope codes + the 18 scales + 14 pad);
// two converter warps turn them into fp16 in place, in the layout of the bf16 form.
constexpr int LAT_RAW = LAT_SLOT / 2;
constexpr int ROPE_RAW = 2048;
constexpr int SMEM8 = SMEM;
constexpr int C8_WARPS = 4;
// The MMA issuing threads' issue rate bounds the kernel (52 MMAs a tile).  A warp shares its
// scheduler with the warps of the same index mod 4; softmax warp 3 serves TMEM lanes 96..127,
// beyond the 80 heads, and is nearly idle, so the bf16 kernel puts the score issuer on warp 7.
// The MXFP8 kernel keeps it on warp 5 beside its converters.
template <bool C8>
constexpr int mma_warp() { return C8 ? 5 : 7; }
// The PV MMAs have their own issuing thread, so that the two chains (S, PV) are issued in
// parallel; they touch disjoint TMEM columns and slots.  bf16: warp 6.  MXFP8: warp 11, on the
// scheduler of the idle softmax warp 3 (warps 6-9 convert, warp 10 is idle).
template <bool C8>
constexpr int pv_warp() { return C8 ? 11 : 6; }
template <bool C8>
constexpr int block_threads() { return C8 ? 384 : 256; }
// The M = 128 score MMA reads 128 rows of each 80-row q~ box: the 48 rows past a box are the
// next box, or (for the last box) the first 6 KB of P.  They only feed unused score rows.
static_assert(P_OFF + 48 * 128 <= LAT_OFF, "q~ box over-read stays in the P buffer");
}  // namespace dsk

struct SkBars {
  float scale[dsk::NH];
  uint64_t q_ready;                               // q~ (TMA part + TMEM part) of a segment
  uint64_t lat_full[dsk::NLAT], lat_empty[dsk::NLAT];
  uint64_t rope_full[dsk::NROPE], rope_empty[dsk::NROPE];
  uint64_t lat_raw[dsk::NLAT], rope_raw[dsk::NROPE];  // MXFP8 cache: raw rows landed (TMA)
  uint64_t s_full, s_free, p_ready, pv_done, seg_done, mma_final;
  uint32_t tmem_base;
};

__device__ __forceinline__ uint8_t* dsk_align(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Key range of query row r: it is new token r % q_len of sequence r / q_len and sees the cache
// rows 0 .. cache_len + r % q_len (the window keeps the last W of them).  (r: the query row,
// not its position in the work list.)
__device__ __forceinline__ void dsk_row_range(const DecAttnParams& p, int r, int* lo, int* hi) {
  const int ql = p.q_len > 1 ? p.q_len : 1;
  const int L = p.cache_len[r / ql] + r % ql;
  *hi = L;
  *lo = p.window > 0 ? max(0, L - p.window + 1) : 0;
}

// One segment: the tiles [g0, g1) of the global list, all in the row at list position r.
struct DskSeg {
  int r, g0, g1;        // list position of the row; global tile range
  int q;                // the query row (token q % q_len of sequence q / q_len)
  int tile0;            // tile index (of TP positions) within the row of global tile g0
  int lo, hi;           // row's key range
};

// Walks the segments of this CTA's range in order; every role walks the same sequence.
struct DskWalk {
  int t, t_end, r;
  __device__ void init(const DecAttnParams& p) {
    // G = min(grid, N) CTAs (a multiple of q_len) share the N tiles, so that no CTA range is
    // empty (the merge kernel relies on it); the CTAs beyond G have nothing to do
    const long long N = p.tstart[p.R];
    const long long G = dec_ctas_used(N, gridDim.x, p.q_len > 1 ? p.q_len : 1);
    if ((long long)blockIdx.x >= G) {
      t = t_end = r = 0;
      return;
    }
    t = int(N * blockIdx.x / G);
    t_end = int(N * (blockIdx.x + 1) / G);
    // the row holding tile t: the largest r with tstart[r] <= t
    int a = 0, b = p.R - 1;
    while (a < b) {
      const int m = (a + b + 1) >> 1;
      if (p.tstart[m] <= t) a = m; else b = m - 1;
    }
    r = a;
  }
  __device__ bool next(const DecAttnParams& p, DskSeg* s) {
    if (t >= t_end) return false;
    while (p.tstart[r + 1] <= t) ++r;
    s->r = r;
    s->q = dec_row_of(r, p.q_len > 1 ? p.q_len : 1, p.n_seq);
    s->g0 = t;
    s->g1 = min(t_end, p.tstart[r + 1]);
    dsk_row_range(p, s->q, &s->lo, &s->hi);
    s->tile0 = s->lo / dsk::TP + (t - p.tstart[r]);
    t = s->g1;
    return true;
  }
};

static_assert(sizeof(SkBars) <= 1024, "barrier block");

// C8: the cache holds MXFP8 rows (mapC: their 128-code latent boxes, mapR: their rope codes and
// scales); 128 more threads (warps 6-9) convert them, and q~, P and the cache tiles are fp16 MMA
// operands instead of bf16.
template <bool C8>
__global__ void __launch_bounds__(dsk::block_threads<C8>(), 1)
    dec_attn_sk_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapC,
                       const __grid_constant__ CUtensorMap mapR, const __grid_constant__ DecAttnParams p,
                       KernelCtl ctl) {
  using namespace dsk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = dsk_align(smem_raw);
  SkBars* bars = reinterpret_cast<SkBars*>(smem + BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ql = p.q_len > 1 ? p.q_len : 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_ready, 5);          // producer's expect_tx + the four softmax warps
    // full: the producer's expect_tx (bf16 tiles), or one arrival per converter warp (C8)
    for (int s = 0; s < NLAT; ++s) {
      mbar_init(&bars->lat_full[s], C8 ? C8_WARPS : 1);
      mbar_init(&bars->lat_empty[s], 1);
      mbar_init(&bars->lat_raw[s], 1);
    }
    for (int s = 0; s < NROPE; ++s) {
      mbar_init(&bars->rope_full[s], C8 ? C8_WARPS : 1);
      mbar_init(&bars->rope_empty[s], 1);
      mbar_init(&bars->rope_raw[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);           // one arrival per softmax warp: S read out of TMEM
    mbar_init(&bars->p_ready, 4);          // one arrival per softmax warp: P written
    mbar_init(&bars->pv_done, 1);
    // (both issuing threads commit to these)
    mbar_init(&bars->seg_done, 2);
    mbar_init(&bars->mma_final, 2);
    fence_mbar_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapC);
    if (C8) tma_prefetch_desc(&mapR);
  }
  if (warp == mma_warp<C8>()) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  DskWalk walk;
  walk.init(p);
  DskSeg sg;

  if (warp == 4) {
    if (lane == 0) {
      // ============================================================ TMA producer
      uint32_t lat_issued = 0, lat_par = 0, rope_issued = 0, rope_par = 0;
      bool q_issued = false;
      bool ok = true;
      int J = 0;            // CTA-local tile counter (over all segments)
      int seg = 0;
      while (ok && walk.next(p, &sg)) {
        const long long crow0 = (long long)(sg.q / ql) * p.cap;
        bool q_done = false;
        auto load_q = [&]() -> bool {
          // the previous segment's score MMAs read the shared q~ boxes until it is done
          if (seg > 0 && !mbar_wait(&bars->seg_done, (seg - 1) & 1, ctl, SITE_DEC_PRODUCER)) return false;
          mbar_expect_tx(&bars->q_ready, 5 * QS_BOX);
          for (int c = 0; c < 5; ++c)
            tma_load_2d(smem + QS_OFF + c * QS_BOX, &mapQ, &bars->q_ready, 256 + 64 * c, sg.q * NH);
          q_issued = true;
          return true;
        };
        const int n_tiles = sg.g1 - sg.g0;
        // the segment's key rows lie in one sequence: [crow0 + lo', crow0 + hi], contiguous
        auto prefetch = [&](int jj) {
          const int pos = (sg.tile0 + jj) * TP;
          const int first = max(pos, sg.lo), last = min(pos + TP - 1, sg.hi);
          if (first <= last)
            l2_prefetch_bulk(static_cast<const uint8_t*>(p.cache) + (crow0 + first) * 1152,
                             uint32_t(last - first + 1) * 1152u);
        };
        for (int jj = 0; jj < PREFETCH_AHEAD && jj < n_tiles; ++jj) prefetch(jj);
        for (int j = 0; j < n_tiles && ok; ++j, ++J) {
          if (PREFETCH_AHEAD > 0 && j + PREFETCH_AHEAD < n_tiles) prefetch(j + PREFETCH_AHEAD);
          const int y = int(crow0 + (long long)(sg.tile0 + j) * TP);
          // the latent units and the rope box (for MXFP8 rows the rope box, which carries the
          // rows' block scales, goes first: the converters need it before any latent unit)
          auto load_lat = [&]() -> bool {
            for (int u = 0; u < 4 && ok; ++u) {
              const int gl = 4 * J + u, s = gl % NLAT;
              const uint32_t ph = (gl / NLAT) & 1;
              if (gl >= NLAT && !mbar_wait(&bars->lat_empty[s], ph ^ 1, ctl, SITE_DEC_PRODUCER)) return false;
              uint8_t* dst = smem + LAT_OFF + s * LAT_SLOT;
              if (C8) {
                // [64 rows][128 codes] of the MXFP8 rows into the slot's upper half
                mbar_expect_tx(&bars->lat_raw[s], LAT_SLOT / 2);
                tma_load_2d(dst + LAT_RAW, &mapC, &bars->lat_raw[s], 128 * u, y);
              } else {
                mbar_expect_tx(&bars->lat_full[s], LAT_SLOT);
                tma_load_2d(dst, &mapC, &bars->lat_full[s], 128 * u, y);
                tma_load_2d(dst + LAT_SLOT / 2, &mapC, &bars->lat_full[s], 128 * u + 64, y);
              }
              lat_issued |= 1u << s;
              lat_par = (lat_par & ~(1u << s)) | (ph << s);
            }
            return true;
          };
          auto load_rope = [&]() -> bool {
            {
              const int s = J % NROPE;
              const uint32_t ph = (J / NROPE) & 1;
              if (J >= NROPE && !mbar_wait(&bars->rope_empty[s], ph ^ 1, ctl, SITE_DEC_PRODUCER)) return false;
              if (C8) {
                // [64 rows][96 bytes]: the rope codes, the 18 block scales and the padding
                mbar_expect_tx(&bars->rope_raw[s], 64 * 96);
                tma_load_2d(smem + ROPE_OFF + s * ROPE_SLOT + ROPE_RAW, &mapR, &bars->rope_raw[s], 512, y);
              } else {
                mbar_expect_tx(&bars->rope_full[s], ROPE_SLOT);
                tma_load_2d(smem + ROPE_OFF + s * ROPE_SLOT, &mapC, &bars->rope_full[s], 512, y);
              }
              rope_issued |= 1u << s;
              rope_par = (rope_par & ~(1u << s)) | (ph << s);
            }
            return true;
          };
          if (C8 ? !(load_rope() && load_lat()) : !(load_lat() && load_rope())) { ok = false; break; }
          // q~ of this segment goes after its first tile: that tile's loads overlap the wait
          // for the previous segment to finish with the shared q~ boxes
          if (!q_done) {
            if (!load_q()) { ok = false; break; }
            q_done = true;
          }
        }
        ++seg;
      }
      for (int s = 0; s < NLAT; ++s)
        if (lat_issued & (1u << s))
          mbar_drain(C8 ? &bars->lat_raw[s] : &bars->lat_full[s], (lat_par >> s) & 1, ctl.err);
      for (int s = 0; s < NROPE; ++s)
        if (rope_issued & (1u << s))
          mbar_drain(C8 ? &bars->rope_raw[s] : &bars->rope_full[s], (rope_par >> s) & 1, ctl.err);
      if (q_issued) mbar_drain(&bars->q_ready, (seg - 1) & 1, ctl.err);
    }
  } else if (warp == mma_warp<C8>()) {
    if (lane == 0) {
      // ============================================================ score (S) issuer
      // Descriptors as (low, high) words; offsets below are in 16-byte units of the low word.
      constexpr uint32_t idesc_s = make_idesc(128, TP, C8 ? 0 : 1, 0, 0);    // fp16 (C8) or bf16
      const uint32_t hi = uint32_t(sdesc_sw128(smem_u32(smem), 16, 1024) >> 32);
      const uint32_t qs_lo = uint32_t(sdesc_sw128(smem_u32(smem + QS_OFF), 16, 1024));
      const uint32_t lat_lo = uint32_t(sdesc_sw128(smem_u32(smem + LAT_OFF), 16, 1024));        // K-major
      const uint32_t rope_lo = uint32_t(sdesc_sw128(smem_u32(smem + ROPE_OFF), 16, 1024));
      const uint32_t tS = tmem + S_COL;
      bool ok = true;
      int J = 0, seg = 0;
      int ls = 0, rs = 0;                      // ring slot of the tile's first latent unit / its rope unit
      uint32_t lph = 0, rph = 0;               // parity of the next full-wait, per slot
      while (ok && walk.next(p, &sg)) {
        if (!mbar_wait(&bars->q_ready, seg & 1, ctl, SITE_DEC_MMA)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; j < sg.g1 - sg.g0; ++j, ++J) {
          // ---- S(J) = q~ C(J)^T, once the softmax has read S(J - 1) out of TMEM: latent dims
          // 0..255 with A in TMEM, 256..511 and rope with A in smem
          if (j > 0 && !mbar_wait(&bars->s_free, (J - 1) & 1, ctl, SITE_DEC_MMA)) { ok = false; break; }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            int s = ls + u;
            if (s >= NLAT) s -= NLAT;
            if (!mbar_wait(&bars->lat_full[s], (lph >> s) & 1, ctl, SITE_DEC_MMA)) { ok = false; break; }
            lph ^= 1u << s;
            tc_fence_after();
            const uint32_t b = lat_lo + uint32_t(s) * (LAT_SLOT / 16);
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
              const int c = 2 * u + bx;             // 64-dim chunk of the latent
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t bd = b + uint32_t(bx * (LAT_SLOT / 32) + kk * 2);
                if (c < 4)
                  mma_ts_w(tS, tmem + QT_COL + (4 * c + kk) * 8, bd, hi, idesc_s, (c | kk) != 0);
                else
                  mma_ss_w(tS, qs_lo + uint32_t((c - 4) * (QS_BOX / 16) + kk * 2), hi, bd, hi, idesc_s, 1u);
              }
            }
          }
          if (!ok) break;
          if (!mbar_wait(&bars->rope_full[rs], (rph >> rs) & 1, ctl, SITE_DEC_MMA)) { ok = false; break; }
          rph ^= 1u << rs;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_w(tS, qs_lo + uint32_t(4 * (QS_BOX / 16) + kk * 2), hi,
                     rope_lo + uint32_t(rs * (ROPE_SLOT / 16) + kk * 2), hi, idesc_s, 1u);
          mma_commit(&bars->s_full);
          mma_commit(&bars->rope_empty[rs]);
          rs = rs + 1 == NROPE ? 0 : rs + 1;
          ls += 4;
          if (ls >= NLAT) ls -= NLAT;
        }
        if (!ok) break;
        mma_commit(&bars->seg_done);
        ++seg;
      }
      mma_commit(&bars->mma_final);
      mbar_drain(&bars->mma_final, 0, ctl.err);
    }
  } else if (warp == pv_warp<C8>()) {
    if (lane == 0) {
      // ============================================================ PV issuer
      // PV(J): O^T += C(J)^T P^T as soon as the softmax has written P(J); the tile's slots are
      // released block by block; the first PV of a segment starts O^T afresh
      constexpr uint32_t idesc_o = make_idesc(128, NH, C8 ? 0 : 1, 1, 0);
      const uint32_t hi = uint32_t(sdesc_sw128(smem_u32(smem), 16, 1024) >> 32);
      const uint32_t p_lo = uint32_t(sdesc_sw128(smem_u32(smem + P_OFF), 16, 1024));
      const uint32_t latv_lo = uint32_t(sdesc_sw128(smem_u32(smem + LAT_OFF), LAT_SLOT / 2, 1024));  // MN-major
      bool ok = true;
      int J = 0;
      while (ok && walk.next(p, &sg)) {
        for (int j = 0; j < sg.g1 - sg.g0; ++j, ++J) {
          if (!mbar_wait(&bars->p_ready, J & 1, ctl, SITE_DEC_MMA)) { ok = false; break; }
          tc_fence_after();
          int s0 = (4 * J) % NLAT;
#pragma unroll
          for (int mb = 0; mb < 4; ++mb) {
            int s = s0 + mb;
            if (s >= NLAT) s -= NLAT;
            const uint32_t a = latv_lo + uint32_t(s) * (LAT_SLOT / 16);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss_w(tmem + O_COL + NH * mb, a + uint32_t(kk * 128), hi, p_lo + uint32_t(kk * 2), hi, idesc_o,
                       (j > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars->lat_empty[s]);
          }
          mma_commit(&bars->pv_done);
        }
        if (!ok) break;
        mma_commit(&bars->seg_done);
      }
      mma_commit(&bars->mma_final);
      mbar_drain(&bars->mma_final, 0, ctl.err);
    }
  } else if (C8 && warp >= 6 && warp < 6 + C8_WARPS) {
    // ============================================================ MXFP8 converters (warps 6-9)
    // Two threads per row (half h of its codes).  Per tile: the rope box first (its bytes hold
    // the row's 18 block scales, which the threads keep for the latent units), then the four
    // latent units, thread h writing fp16 box h of the unit (64 of its 128 dims); each unit: all
    // 128 threads read their raw half rows, meet at a named barrier (the fp16 output overwrites
    // the raw bytes), convert E4M3 x 2^k -> fp16 into the 128-byte-swizzled K-major boxes and
    // publish the slot.  Rows outside the row's key range become zeros, so an unwritten cache
    // tail (NaN codes or scales) never reaches the MMAs.
    const int c_id = threadIdx.x - 192;
    const int r = c_id >> 1, hh = c_id & 1;
    const int sw = r & 7;
    bool ok = true;
    int J = 0;
    bool fp16_bad = false;
    // 16 E4M3 codes (one uint4) times 2^k -> 16 fp16 values (two uint4)
    // (rows outside the key range are converted too, then replaced by zeros: only valid rows
    // may report an fp16 range error)
    // For a scale 2^k with k in [-14, 7] the product E4M3 x 2^k is an exact fp16 (at most
    // 448 2^7 < 65504; the smallest, 2^-9 2^-14, is a multiple of the fp16 subnormal step 2^-24),
    // so it is one fp16x2 multiply; other scales go through fp32 with a saturating check.
    auto convert16 = [&](const uint4 c, int k, uint4& o0, uint4& o1, bool valid) {
      bool bad = false;
      const uint32_t w[4] = {c.x, c.y, c.z, c.w};
      uint32_t h[8];
      if (k >= -14 && k <= 7) {
        const uint32_t sh = uint32_t(k + 15) << 10;
        const __half2 s2 = __halves2half2(__ushort_as_half(uint16_t(sh)), __ushort_as_half(uint16_t(sh)));
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            uint32_t x = f16x2_from_e4m3x2(uint16_t(w[i] >> (16 * e)));
            __half2 v = __hmul2(*reinterpret_cast<__half2*>(&x), s2);
            h[2 * i + e] = *reinterpret_cast<uint32_t*>(&v);
          }
        }
      } else {
        const float s = exp2i(k);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint32_t x = f16x2_from_e4m3x2(uint16_t(w[i] >> (16 * e)));
            const float lo = __half2float(__ushort_as_half(uint16_t(x & 0xFFFFu))) * s;
            const float hi = __half2float(__ushort_as_half(uint16_t(x >> 16))) * s;
            h[2 * i + e] = pack_half2_sat(lo, hi, bad);
          }
        }
      }
      fp16_bad |= bad && valid;
      o0 = valid ? make_uint4(h[0], h[1], h[2], h[3]) : make_uint4(0u, 0u, 0u, 0u);
      o1 = valid ? make_uint4(h[4], h[5], h[6], h[7]) : make_uint4(0u, 0u, 0u, 0u);
    };
    while (ok && walk.next(p, &sg)) {
      for (int j = 0; j < sg.g1 - sg.g0 && ok; ++j, ++J) {
        const int pos = (sg.tile0 + j) * TP + r;
        const bool valid = pos >= sg.lo && pos <= sg.hi;
        // ---- rope box and scales
        const int rs = J % NROPE;
        const bool wr = mbar_wait(&bars->rope_raw[rs], (J / NROPE) & 1, ctl, SITE_DEC_CONVERT);
        uint8_t* rslot = smem + ROPE_OFF + rs * ROPE_SLOT;
        const uint8_t* raw = rslot + ROPE_RAW + r * 96;
        uint4 rc[2];                          // rope codes 32 hh .. 32 hh + 31
#pragma unroll
        for (int i = 0; i < 2; ++i) rc[i] = *reinterpret_cast<const uint4*>(raw + 32 * hh + 16 * i);
        const uint4 sc = *reinterpret_cast<const uint4*>(raw + 64);          // scales of blocks 0..15
        const uint32_t sc2 = *reinterpret_cast<const uint32_t*>(raw + 80);   // blocks 16, 17
        // every raw row read before any is overwritten (and a failed wait stops both warps)
        if (named_bar_or(2, 32 * C8_WARPS, !wr)) { ok = false; break; }
        {
          const int sr = int((sc2 >> (8 * hh)) & 0xFFu) - 127;     // block 16 + hh
#pragma unroll
          for (int i = 0; i < 2; ++i) {       // codes 32 hh + 16 i ..: chunks 4 hh + 2 i, + 1
            const int ch = 4 * hh + 2 * i;
            uint4 o0, o1;
            convert16(rc[i], sr, o0, o1, valid);
            *reinterpret_cast<uint4*>(rslot + r * 128 + ((ch ^ sw) << 4)) = o0;
            *reinterpret_cast<uint4*>(rslot + r * 128 + (((ch + 1) ^ sw) << 4)) = o1;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->rope_full[rs]);
        // ---- latent units
        const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll 1
        for (int u = 0; u < 4; ++u) {
          const int gl = 4 * J + u, s = gl % NLAT;
          const bool wl = mbar_wait(&bars->lat_raw[s], (gl / NLAT) & 1, ctl, SITE_DEC_CONVERT);
          uint8_t* slot = smem + LAT_OFF + s * LAT_SLOT;
          uint4 c[4];                         // codes 64 hh .. 64 hh + 63 of the unit
#pragma unroll
          for (int i = 0; i < 4; ++i) c[i] = *reinterpret_cast<const uint4*>(slot + LAT_RAW + r * 128 + 64 * hh + 16 * i);
          if (named_bar_or(2, 32 * C8_WARPS, !wl)) { ok = false; break; }
          // codes 64 hh + 16 i ..: block 4 u + 2 hh + i / 2; box hh, chunks 2 i, 2 i + 1
          uint8_t* box = slot + hh * (LAT_SLOT / 2) + r * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int sk = int((scw[u] >> (8 * (2 * hh + (i >> 1)))) & 0xFFu) - 127;
            uint4 o0, o1;
            convert16(c[i], sk, o0, o1, valid);
            *reinterpret_cast<uint4*>(box + (((2 * i) ^ sw) << 4)) = o0;
            *reinterpret_cast<uint4*>(box + (((2 * i + 1) ^ sw) << 4)) = o1;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->lat_full[s]);
        }
      }
    }
    if (fp16_bad && p.err) atomicCAS(p.err, 0, SITE_FP16_RANGE);
  } else if (warp < 4) {
    // ============================================================ softmax / epilogue (warps 0-3)
    const int q = warp;                      // TMEM lane quarter
    const int h = 32 * q + lane;             // head of this thread (h < 80), latent row in O^T
    const bool hv = h < NH;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    uint8_t* P = smem + P_OFF;
    bool ok = true;
    int J = 0, seg = 0;
    auto group_ok = [&](bool w) { return !named_bar_or(1, 128, !w); };
    while (ok && walk.next(p, &sg)) {
      // ---- q~ dims 0..255 of this row into TMEM (lane = head, two dims per column)
      // (from the second segment on, the previous segment's MMAs are complete and its partial
      // was read out at the end of the loop below)
      if (q < 3) {
        uint32_t v[32];
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.qt) +
                                                          ((long long)sg.q * NH + (hv ? h : 0)) * 576);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 w = hv ? src[8 * c + k] : make_uint4(0u, 0u, 0u, 0u);
            v[4 * k] = w.x; v[4 * k + 1] = w.y; v[4 * k + 2] = w.z; v[4 * k + 3] = w.w;
          }
          GDLA_TMEM_ST32(tmem + QT_COL + 32 * c + lane_off, v);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_ready);

      float m_ref = -INFINITY;
      float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;   // row sum, in four partials
      bool carried_fail = false;                          // a wait of the last tile expired
      for (int j = 0; j < sg.g1 - sg.g0; ++j, ++J) {
        // (warp-uniform: the TMEM load below is a warp-collective instruction)
        const bool w = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, J & 1, ctl, SITE_DEC_SOFTMAX));
        tc_fence_after();
        const int pos0 = (sg.tile0 + j) * TP;
        const int a = sg.lo - pos0, bnd = sg.hi - pos0;   // valid columns a .. bnd
        const bool edge = a > 0 || bnd < TP - 1;           // uniform: a boundary tile of the row
        float v[TP];
        float mt = -INFINITY;
        if (q < 3 && w) {
          uint32_t u[TP];
          GDLA_TMEM_LD32(tmem + S_COL + lane_off, u);
          GDLA_TMEM_LD32(tmem + S_COL + 32 + lane_off, (u + 32));
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < TP; ++c) v[c] = __uint_as_float(u[c]);
        }
        // S is in registers: the MMA issuer may overwrite it with the next tile's scores
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        if (q < 3) {
          if (edge) {
#pragma unroll
            for (int c = 0; c < TP; ++c) v[c] = (c >= a && c <= bnd) ? v[c] : -INFINITY;
          }
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            m8[k] = fmax3f(fmax3f(v[8 * k], v[8 * k + 1], v[8 * k + 2]), fmax3f(v[8 * k + 3], v[8 * k + 4], v[8 * k + 5]),
                           fmaxf(v[8 * k + 6], v[8 * k + 7]));
          mt = fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * p.scale_log2;
        }
        // the one barrier of the common path: does any head need its reference maximum moved
        // (or did any wait expire)?
        const bool need = hv && mt > m_ref + RESCALE_THRESHOLD;
        if (named_bar_or(1, 128, need || !w || carried_fail)) {
          if (named_bar_or(1, 128, !w || carried_fail)) { ok = false; break; }
          // O^T must hold PV(J - 1) before it is rescaled (PV(J) comes after this tile's P)
          bool w2 = j == 0 || mbar_wait(&bars->pv_done, (J - 1) & 1, ctl, SITE_DEC_SOFTMAX);
          if (named_bar_or(1, 128, !w2)) { ok = false; break; }
          tc_fence_after();
          if (hv) {
            const float mn = need ? mt : m_ref;
            const float sc = need ? ex2_approx(m_ref - mn) : 1.f;   // 2^-inf = 0 on the first tile
            ls0 *= sc; ls1 *= sc; ls2 *= sc; ls3 *= sc;
            m_ref = mn;
            bars->scale[h] = sc;
          }
          named_bar_sync(1, 128);
          if (j > 0) {
#pragma unroll 1
            for (int c = 0; c < 4 * 5; ++c) {
              const uint32_t tO = tmem + O_COL + NH * (c / 5) + 16 * (c % 5) + lane_off;
              uint32_t o[16];
              GDLA_TMEM_LD16(tO, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e)
                o[e] = __float_as_uint(__uint_as_float(o[e]) * bars->scale[16 * (c % 5) + e]);
              GDLA_TMEM_ST16(tO, o);
            }
            tmem_st_wait();
          }
          named_bar_sync(1, 128);
        }
        // P has one buffer: PV(J - 1) must have read it (earlier segments' PVs are complete)
        const bool w3 = j == 0 || mbar_wait(&bars->pv_done, (J - 1) & 1, ctl, SITE_DEC_SOFTMAX);
        carried_fail = !w3;
        if (!C8 && edge && bnd < TP - 1) {
          // rows past the row's last key: zero them in the four latent slots before the PV (the
          // MXFP8 converters have written such rows as zeros already)
          const int r0 = bnd + 1;
          const int nbytes = (TP - r0) * 128;
#pragma unroll 1
          for (int bx = 0; bx < 8; ++bx) {
            uint8_t* box = smem + LAT_OFF + ((4 * J + bx / 2) % NLAT) * LAT_SLOT + (bx & 1) * (LAT_SLOT / 2);
            for (int o = (q * 32 + lane) * 16; o < nbytes; o += 128 * 16)
              *reinterpret_cast<uint4*>(box + r0 * 128 + o) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        // numerators 2^(s scale - m) (every fourth pair on the FMA pipe), rounded to bf16, one
        // 128-byte row of P per head in the 128-byte-swizzled K-major layout of the PV's B operand
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
        uint8_t* row = P + h * 128;
        if (hv && w3) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 8 * k + 2 * e;
              float x0, x1, p0, p1;
              ffma2(x0, x1, v[c], v[c + 1], p.scale_log2, neg_m);
              if (e == 3) {
                exp2_poly2(x0, x1, p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              if (edge) {
                p0 = (c >= a && c <= bnd) ? p0 : 0.f;
                p1 = (c + 1 >= a && c + 1 <= bnd) ? p1 : 0.f;
              }
              // the row sum adds the rounded values the PV multiplies (weights summing to 1)
              float r0, r1;
              if (C8) {
                pk[e] = pack_half2(p0, p1);
                r0 = __half2float(__ushort_as_half(uint16_t(pk[e] & 0xFFFFu)));
                r1 = __half2float(__ushort_as_half(uint16_t(pk[e] >> 16)));
              } else {
                pk[e] = pack_bf162(p0, p1);
                r0 = __uint_as_float(pk[e] << 16);
                r1 = __uint_as_float(pk[e] & 0xFFFF0000u);
              }
              if (e & 1) fadd2(ls2, ls3, r0, r1); else fadd2(ls0, ls1, r0, r1);
            }
            *reinterpret_cast<uint4*>(row + ((k ^ (h & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_ready);
      }
      const float l_sum = (ls0 + ls1) + (ls2 + ls3);
      if (!ok) break;
      // ---- segment partial: (m_h, l_h) and O^T, to slot blockIdx.x + r
      const bool w = mbar_wait(&bars->seg_done, seg & 1, ctl, SITE_DEC_SOFTMAX);
      if (!group_ok(w && !carried_fail)) { ok = false; break; }
      tc_fence_after();
      const long long slot = (long long)blockIdx.x + sg.r;
      if (hv) {
        float* ml = p.ml + (slot * NH + h) * 2;
        ml[0] = m_ref;
        ml[1] = l_sum;
      }
#pragma unroll 1
      for (int mb = 0; mb < 4; ++mb) {
        const uint32_t tO = tmem + O_COL + NH * mb + lane_off;
        uint32_t o[NH];
        GDLA_TMEM_LD32(tO, o);
        GDLA_TMEM_LD32(tO + 32, (o + 32));
        GDLA_TMEM_LD16(tO + 64, (o + 64));
        tmem_ld_wait();
        float* dst = p.part + slot * NH * 512 + 128 * mb + h;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) dst[(long long)hh * 512] = __uint_as_float(o[hh]);
      }
      tc_fence_before();
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == mma_warp<C8>()) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Tile prefix over the query rows in list order (dec_list_pos): tstart[l] = tiles of the rows
// before list position l, tstart[R] = all tiles.  A row whose cache_len entry is outside
// [0, cap - q_len] gets no tiles (its output is zero) and the error word records
// SITE_BAD_CACHE_LEN.  One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) dec_sched_kernel(const int* __restrict__ cache_len, int R, int q_len,
                                                         int cap, int window, int* __restrict__ tstart,
                                                         int* err) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ql = q_len > 1 ? q_len : 1;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < R; base += blockDim.x) {
    const int l = base + threadIdx.x;           // list position (token-major order)
    int n = 0;
    if (l < R) {
      const int r = dec_row_of(l, ql, R / ql);
      const int L0 = cache_len[r / ql];
      if (L0 < 0 || L0 > cap - ql) {
        if (r % ql == 0) atomicCAS(err, 0, SITE_BAD_CACHE_LEN);
      } else {
        const int L = L0 + r % ql;
        const int lo = window > 0 ? max(0, L - window + 1) : 0;
        n = L / dsk::TP - lo / dsk::TP + 1;
      }
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int s = lane < int(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;
    }
    __syncthreads();
    const int incl = x + (warp > 0 ? wsum[warp - 1] : 0) + carry;
    if (l < R) tstart[l] = incl - n;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) tstart[R] = carry;
}

int launch_dec_sched(const DecAttnParams& p, cudaStream_t st) {
  dec_sched_kernel<<<1, 1024, 0, st>>>(p.cache_len, p.R, p.q_len, p.cap, p.window, p.tstart, p.err);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

int launch_dec_attn_tc(const DecAttnParams& p, KernelCtlHost ctl, cudaStream_t st) {
  CUtensorMap mq, mc, mr;
  const bool c8 = p.cache_fp8 != 0;
  if (make_tmap_2d(&mq, c8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.qt, 576,
                   (uint64_t)p.R * dsk::NH, 576 * 2, 64, dsk::NH, CU_TENSOR_MAP_SWIZZLE_128B))
    return -3;
  if (c8) {
    // MXFP8 rows of 608 bytes: [64 rows][128 codes] latent boxes, [64 rows][96 bytes] rope + scales
    if (make_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.cache, FP8_ROW_BYTES, (uint64_t)p.n_seq * p.cap,
                     FP8_ROW_BYTES, 128, dsk::TP, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        make_tmap_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.cache, FP8_ROW_BYTES, (uint64_t)p.n_seq * p.cap,
                     FP8_ROW_BYTES, 96, dsk::TP, CU_TENSOR_MAP_SWIZZLE_NONE))
      return -3;
  } else {
    if (make_tmap_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.cache, 576, (uint64_t)p.n_seq * p.cap, 576 * 2,
                     64, dsk::TP, CU_TENSOR_MAP_SWIZZLE_128B))
      return -3;
    mr = mc;
  }
  KernelCtl kc{ctl.err, ctl.limit_ns};
  if (c8) {
    if (cudaFuncSetAttribute(dec_attn_sk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dsk::SMEM8) != cudaSuccess)
      return -4;
    dec_attn_sk_kernel<true><<<p.n_ctas, dsk::block_threads<true>(), dsk::SMEM8, st>>>(mq, mc, mr, p, kc);
  } else {
    if (cudaFuncSetAttribute(dec_attn_sk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dsk::SMEM) != cudaSuccess)
      return -4;
    dec_attn_sk_kernel<false><<<p.n_ctas, dsk::block_threads<false>(), dsk::SMEM, st>>>(mq, mc, mr, p, kc);
  }
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

// CTAs of the decode attention: one per SM (its shared memory and 512 TMEM columns fill one).
int decode_cta_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n < DEC_MAX_CTAS ? n : DEC_MAX_CTAS;
}

}  // namespace gdla
