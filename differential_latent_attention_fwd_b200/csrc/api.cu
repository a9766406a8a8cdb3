// C ABI of the GDLA forward pass: argument validation, workspace carving and the launch
// sequence of the prefill and absorbed-decode paths (declared in include/gdla.h).
#include "../../include/gdla.h"
#include "gdla_common.cuh"
#include "gdla_decode.h"
#include "gdla_internal.h"

#include <math.h>
#include <string.h>

#include <mutex>

namespace gdla {

// Device error word written by bounded waits (one instance per device that loads the library).
__device__ int g_device_error = 0;

static unsigned long long g_wait_limit_ns = 2000000000ull;
static cudaEvent_t g_stage_ev[8];
static int g_n_stage_ev = 0;
static unsigned long long g_launches = 0;

static void stage(int i, cudaStream_t st) {
  if (i < g_n_stage_ev) cudaEventRecord(g_stage_ev[i], st);
}
// Every launch_* helper enqueues exactly one kernel; returns true on failure.
static bool launch_failed(int rc) {
  if (rc == 0) ++g_launches;
  return rc != 0;
}
}  // namespace gdla
namespace gdla {
void count_extra_launch() { ++g_launches; }
static const uint32_t kAbsorbedMagic = 0x47444C41u;  // "GDLA"

static int error_word(int** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return GDLA_ERR_CUDA;
  *out = static_cast<int*>(p);
  return GDLA_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_config(const gdla_config_t* c) {
  if (!c) return GDLA_ERR_INVALID_ARG;
  if (c->d_nope != 128 || c->d_rope != 64 || c->d_v != 128) return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (c->q_rank != 1024 || c->kv_rank != 512) return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (c->n_noise <= 0 || c->n_signal != 4 * c->n_noise || c->n_kv_heads != c->n_noise)
    return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (c->n_noise > 16) return GDLA_ERR_UNSUPPORTED_SHAPE;  // decode keeps 80 heads per CTA
  if (c->d_model <= 0 || c->d_model % 64 != 0) return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (c->window < 0 || !(c->rope_theta > 0.f) || !(c->rms_eps >= 0.f)) return GDLA_ERR_INVALID_ARG;
  return GDLA_OK;
}

static int check_weights(const gdla_weights_t* w) {
  if (!w || !w->W_aQ || !w->W_bQ || !w->W_aKV || !w->W_bKV || !w->W_lambda || !w->W_G || !w->W_O)
    return GDLA_ERR_INVALID_ARG;
  const void* ps[] = {w->W_aQ, w->W_bQ, w->W_aKV, w->W_bKV, w->W_lambda, w->W_G, w->W_O};
  for (const void* p : ps)
    if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  if ((w->g_q && !aligned16(w->g_q)) || (w->g_kv && !aligned16(w->g_kv))) return GDLA_ERR_INVALID_ARG;
  return GDLA_OK;
}

// ---------------------------------------------------------------- workspace layout
enum { WS_D1, WS_CQ, WS_LATENT, WS_LAM, WS_QQ, WS_G, WS_KV, WS_ONOISE, WS_DG, WS_KR16, WS_SPLITK,
       WS_VL_POS, WS_VL_UNITS, WS_VL_COUNT, WS_DSCHED, WS_N };

// Packed documents: bounds of the attention schedule for `total` tokens in `n_docs` documents
// (sum over documents of ceil(len / R) <= ceil(total / R) + n_docs, R = ATTN_UNIT_ROWS).  The
// workspace is sized for n_docs = total; the grid uses the actual document count.
static int varlen_max_blocks(long long total) { return int((total + ATTN_UNIT_ROWS - 1) / ATTN_UNIT_ROWS); }
static int varlen_max_units(long long total, long long n_docs) {
  return int(varlen_max_blocks(total) + (n_docs < total ? n_docs : total));
}

// fp32 scratch of the split-K projections of a decode step (skinny M = B products).
static long long decode_splitk_floats(const gdla_config_t* c, int B) {
  const int nH = c->n_signal + c->n_noise;
  const int shapes[3][2] = {{c->q_rank + c->kv_rank + c->d_rope + c->n_signal, c->d_model},
                            {nH * (c->d_nope + c->d_rope) + c->n_signal * c->d_v, c->q_rank},
                            {c->d_model, c->n_signal * c->d_v}};
  long long m = 0;
  for (auto& sh : shapes) {
    const long long f = (long long)gemm_splitk_count(B, sh[0], sh[1]) * B * sh[0];
    if (f > m) m = f;
  }
  return m;
}


static void layout(const gdla_config_t* c, int B, int T, int mode, size_t off[WS_N + 1]) {
  const long long M = mode == GDLA_MODE_DECODE ? (long long)B : (long long)B * T;
  const int nH = c->n_signal + c->n_noise;
  const long long qq = (long long)nH * (c->d_nope + c->d_rope);
  const long long d1 = c->q_rank + c->kv_rank + c->d_rope + c->n_signal;
  size_t sz[WS_N];
  sz[WS_D1] = M * d1 * 4;
  sz[WS_CQ] = M * c->q_rank * 2;
  sz[WS_LAM] = M * c->n_signal * 4;
  sz[WS_G] = M * (long long)c->n_signal * c->d_v * 2;
  sz[WS_DG] = M * (long long)c->n_signal * c->d_v * 2;
  sz[WS_VL_POS] = sz[WS_VL_UNITS] = sz[WS_VL_COUNT] = sz[WS_DSCHED] = 0;
  if (mode == GDLA_MODE_VARLEN) {
    sz[WS_VL_POS] = M * 4;
    sz[WS_VL_UNITS] = (size_t)varlen_max_units(M, M) * 16;
    sz[WS_VL_COUNT] = (size_t)(1 + 2 * varlen_max_blocks(M)) * 4;
  }
  if (mode == GDLA_MODE_PREFILL || mode == GDLA_MODE_VARLEN || mode == GDLA_MODE_CONTEXT) {
    sz[WS_LATENT] = M * (c->kv_rank + c->d_rope) * 2;
    sz[WS_QQ] = M * qq * 2;
    sz[WS_KV] = M * (long long)c->n_kv_heads * (c->d_nope + c->d_v) * 2;
    sz[WS_ONOISE] = ((M + 31) / 32 * 32) * (long long)c->n_noise * c->d_v * 4;   // 32-row blocks
    sz[WS_KR16] = M * c->d_rope * 2;
    sz[WS_SPLITK] = 0;
  } else {
    // the attention's segments: one partial slot per (CTA, row) pair that can meet
    const long long slots = (long long)decode_cta_count() + M;
    sz[WS_LATENT] = 0;                                               // unused by decode
    sz[WS_QQ] = M * (qq + (long long)c->n_signal * c->d_v) * 4;      // fp32 q^C | q^R | G
    sz[WS_G] = 0;                                                    // (G sits in the WS_QQ rows)
    sz[WS_KV] = M * (long long)nH * (c->kv_rank + c->d_rope) * 2;    // q~ rows
    sz[WS_ONOISE] = slots * nH * c->kv_rank * 4;                     // segment partials
    sz[WS_KR16] = slots * nH * 2 * 4;                                // segment (max, sum)
    sz[WS_SPLITK] = decode_splitk_floats(c, B) * 4;
    sz[WS_DSCHED] = (M + 1) * 4;                                     // tile prefix over the rows
  }
  size_t o = 0;
  for (int i = 0; i < WS_N; ++i) {
    off[i] = o;
    o += (sz[i] + 255) & ~size_t(255);
  }
  off[WS_N] = o;
}

// Shared with the other translation units of the library (same error word, same bound).
int shared_kernel_ctl(KernelCtlHost* out) {
  int* err;
  const int rc = error_word(&err);
  if (rc) return rc;
  out->err = err;
  out->limit_ns = g_wait_limit_ns;
  return GDLA_OK;
}

// Packed documents: cu_seqlens on the device; the latent rows go to latent_out (packed order).
struct VarlenArgs {
  const int* cu_seqlens;
  int n_docs;
  void* latent_out;
};

// a1 on token rows [r0, r1): [x W_aQ | x W_aKV | x W_lambda] in fp32 into D1 rows r0..r1-1.
static int down_proj_rows(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x,
                          float* D1, int pos_T, long long r0, long long r1, KernelCtlHost ctl,
                          cudaStream_t st) {
  const int ld1 = cfg->q_rank + cfg->kv_rank + cfg->d_rope + cfg->n_signal;
  const int M = int(r1 - r0);
  if (M <= 0) return GDLA_OK;
  const void* xr = static_cast<const __nv_bfloat16*>(x) + r0 * cfg->d_model;
  float* D = D1 + r0 * ld1;
  GemmEpi ep{};
  ep.ldc = ld1; ep.out_type = OUT_F32; ep.M = M; ep.rope_lo = ep.rope_hi = 0; ep.pos_T = pos_T;
  ep.C = D; ep.N = cfg->q_rank;
  if (launch_failed(launch_gemm(xr, cfg->d_model, w->W_aQ, cfg->q_rank, false, M, cfg->q_rank, cfg->d_model, ep, ctl, st)))
    return GDLA_ERR_LAUNCH;
  ep.C = D + cfg->q_rank; ep.N = cfg->kv_rank + cfg->d_rope;
  if (launch_failed(launch_gemm(xr, cfg->d_model, w->W_aKV, ep.N, false, M, ep.N, cfg->d_model, ep, ctl, st)))
    return GDLA_ERR_LAUNCH;
  ep.C = D + cfg->q_rank + cfg->kv_rank + cfg->d_rope; ep.N = cfg->n_signal;
  if (launch_failed(launch_gemm(xr, cfg->d_model, w->W_lambda, ep.N, false, M, ep.N, cfg->d_model, ep, ctl, st)))
    return GDLA_ERR_LAUNCH;
  return GDLA_OK;
}

// a5 on token rows [r0, r1): y = Dg W^O.
static int out_proj_rows(const gdla_config_t* cfg, const gdla_weights_t* w, const void* Dg, void* y,
                         int pos_T, long long r0, long long r1, KernelCtlHost ctl, cudaStream_t st) {
  const int M = int(r1 - r0);
  if (M <= 0) return GDLA_OK;
  const int kdim = cfg->n_signal * cfg->d_v;
  GemmEpi eo{};
  eo.C = static_cast<__nv_bfloat16*>(y) + r0 * cfg->d_model; eo.ldc = cfg->d_model;
  eo.out_type = OUT_BF16; eo.M = M; eo.N = cfg->d_model; eo.pos_T = pos_T;
  if (launch_failed(launch_gemm(static_cast<const __nv_bfloat16*>(Dg) + r0 * kdim, kdim, w->W_O,
                                cfg->d_model, false, M, cfg->d_model, kdim, eo, ctl, st)))
    return GDLA_ERR_LAUNCH;
  return GDLA_OK;
}

// a2 + a3 on token rows [r0, r1) of B sequences of T tokens (no key prefix, no packed
// documents): norms, rotary key, lambda and latent rows, then q^C | rotated q^R, gate logits and
// K^C | V of those rows.
static int norm_up_rows(const gdla_config_t* cfg, const gdla_weights_t* w, uint8_t* ws,
                        const size_t* off, int T, long long r0, long long r1, const RopeTable& rope,
                        int* err, KernelCtlHost ctl, cudaStream_t st) {
  const int M = int(r1 - r0);
  if (M <= 0) return GDLA_OK;
  const int nH = cfg->n_signal + cfg->n_noise;
  const int ld1 = cfg->q_rank + cfg->kv_rank + cfg->d_rope + cfg->n_signal;
  const int row_w = cfg->kv_rank + cfg->d_rope;
  const int nqq = nH * (cfg->d_nope + cfg->d_rope);
  const int ldg = cfg->n_signal * cfg->d_v;
  const int nkv = cfg->n_kv_heads * (cfg->d_nope + cfg->d_v);
  __nv_bfloat16* cQ = reinterpret_cast<__nv_bfloat16*>(ws + off[WS_CQ]) + r0 * cfg->q_rank;
  __nv_bfloat16* latent = reinterpret_cast<__nv_bfloat16*>(ws + off[WS_LATENT]) + r0 * row_w;
  NormParams np{};
  np.D1 = reinterpret_cast<float*>(ws + off[WS_D1]) + r0 * ld1; np.ld1 = ld1; np.M = M;
  np.q_rank = cfg->q_rank; np.kv_rank = cfg->kv_rank; np.n_signal = cfg->n_signal;
  np.g_q = w->g_q; np.g_kv = w->g_kv; np.eps = cfg->rms_eps;
  np.cQ = cQ; np.latent = latent;
  np.kR16 = reinterpret_cast<__half*>(ws + off[WS_KR16]) + r0 * cfg->d_rope;
  np.lam = reinterpret_cast<float*>(ws + off[WS_LAM]) + r0 * cfg->n_signal;
  np.pos_T = T; np.row_off = int(r0); np.rope = rope; np.err = err;
  if (launch_failed(launch_norm_rope(np, st))) return GDLA_ERR_LAUNCH;
  GemmEpi eq{};
  eq.C = reinterpret_cast<__half*>(ws + off[WS_QQ]) + r0 * nqq; eq.ldc = nqq; eq.out_type = OUT_F16;
  eq.M = M; eq.N = nqq; eq.rope_lo = nH * cfg->d_nope; eq.rope_hi = nqq; eq.pos_T = T;
  eq.row_off = int(r0); eq.rope = rope;
  if (launch_failed(launch_gemm(cQ, cfg->q_rank, w->W_bQ, nqq, false, M, nqq, cfg->q_rank, eq, ctl, st)))
    return GDLA_ERR_LAUNCH;
  GemmEpi eg{};
  eg.C = reinterpret_cast<__nv_bfloat16*>(ws + off[WS_G]) + r0 * ldg; eg.ldc = ldg; eg.out_type = OUT_BF16;
  eg.M = M; eg.N = ldg; eg.pos_T = T;
  if (launch_failed(launch_gemm(cQ, cfg->q_rank, w->W_G, ldg, false, M, ldg, cfg->q_rank, eg, ctl, st)))
    return GDLA_ERR_LAUNCH;
  GemmEpi ekv{};
  ekv.C = reinterpret_cast<__half*>(ws + off[WS_KV]) + r0 * nkv; ekv.ldc = nkv; ekv.out_type = OUT_F16;
  ekv.M = M; ekv.N = nkv; ekv.pos_T = T;
  if (launch_failed(launch_gemm(latent, row_w, w->W_bKV, nkv, false, M, nkv, cfg->kv_rank, ekv, ctl, st)))
    return GDLA_ERR_LAUNCH;
  return GDLA_OK;
}

// Host-buffer prefill: x arrives and y leaves in row pieces on two copy streams; the
// row-separable stages before the attention (a1 - a3) of a piece start as soon as it has
// landed, and each piece of y leaves as soon as its output projection is done.  Null = the
// whole-buffer device path.
struct HostPipeArgs {
  const void* x_host;
  void* y_host;
  int n_pieces;
  cudaStream_t h2d, d2h;
  cudaEvent_t* ev;            // >= 2 * n_pieces + 2 events
};

// A key prefix: the latent rows of the n_prefix tokens that precede x in its sequence.
struct ContextArgs {
  const void* prefix_latent;   // [n_prefix, kv_rank + d_rope] bf16
  int n_prefix;
  int pos_offset;              // position of the first local token (>= n_prefix)
  void* latent_out;            // [T, kv_rank + d_rope] bf16 for the local tokens, or null
};

// Prefill body shared by equal-length batches (vl == ctx == nullptr), packed documents (vl; B =
// 1, T = all tokens), and one sequence chunk after a key prefix (ctx; B = 1).  With latent_only
// it stops after the latent rows (written to ctx->latent_out).  Arguments are already
// validated; off is the workspace layout.
static int prefill_impl(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x, int B,
                        int T, void* y, void* kv_cache_out, int cache_cap, uint8_t* ws,
                        const size_t* off, cudaStream_t st, const VarlenArgs* vl,
                        const ContextArgs* ctx = nullptr, bool latent_only = false,
                        const HostPipeArgs* hp = nullptr) {
  int rc;
  int* err;
  if ((rc = error_word(&err))) return rc;
  KernelCtlHost ctl{err, g_wait_limit_ns};
  float* D1 = reinterpret_cast<float*>(ws + off[WS_D1]);
  void* cQ = ws + off[WS_CQ];
  void* latent = ws + off[WS_LATENT];
  float* lam = reinterpret_cast<float*>(ws + off[WS_LAM]);
  void* QQ = ws + off[WS_QQ];
  void* G = ws + off[WS_G];
  void* KV = ws + off[WS_KV];
  float* On = reinterpret_cast<float*>(ws + off[WS_ONOISE]);
  void* Dg = ws + off[WS_DG];
  void* kR16 = ws + off[WS_KR16];
  const int M = B * T;
  const int nH = cfg->n_signal + cfg->n_noise;
  const int ld1 = cfg->q_rank + cfg->kv_rank + cfg->d_rope + cfg->n_signal;
  const int row_w = cfg->kv_rank + cfg->d_rope;            // latent row: c_bar | rotated k^R
  const int n_pre = ctx ? ctx->n_prefix : 0;               // key rows before the local tokens
  RopeTable rope;
  fill_rope_table(&rope, cfg->d_rope, cfg->rope_theta);

  stage(0, st);
  // packed documents: per-token positions and the attention schedule
  const int* positions = nullptr;
  const int4* units = nullptr;
  const int* n_units = nullptr;
  int max_units = 0;
  if (vl) {
    int* pos = reinterpret_cast<int*>(ws + off[WS_VL_POS]);
    int4* un = reinterpret_cast<int4*>(ws + off[WS_VL_UNITS]);
    int* cnt = reinterpret_cast<int*>(ws + off[WS_VL_COUNT]);
    max_units = varlen_max_units(M, vl->n_docs);
    const int max_c = varlen_max_blocks(M);
    if (launch_failed(launch_varlen_schedule(vl->cu_seqlens, vl->n_docs, M, pos, un, cnt, max_units,
                                             cnt + 1, cnt + 1 + max_c, max_c, err, st)))
      return GDLA_ERR_LAUNCH;
    g_launches += 3;  // the schedule is four kernels
    positions = pos;
    units = un;
    n_units = cnt;
    if (vl->latent_out) latent = vl->latent_out;
  }

  // a1: [x W_aQ | x W_aKV | x W_lambda] in fp32 (with host buffers: piece by piece as x lands)
  if (hp) {
    const long long piece = (M + hp->n_pieces - 1) / hp->n_pieces;
    // the copies must not overtake earlier work on the caller's stream (the workspace may be busy)
    if (cudaEventRecord(hp->ev[0], st) != cudaSuccess || cudaStreamWaitEvent(hp->h2d, hp->ev[0], 0) != cudaSuccess)
      return GDLA_ERR_CUDA;
    for (int k = 0; k < hp->n_pieces; ++k) {
      const long long r0 = k * piece, r1 = r0 + piece < M ? r0 + piece : M;
      if (r0 >= r1) break;
      const size_t bytes = size_t(r1 - r0) * cfg->d_model * 2, off_b = size_t(r0) * cfg->d_model * 2;
      if (cudaMemcpyAsync(static_cast<uint8_t*>(const_cast<void*>(x)) + off_b,
                          static_cast<const uint8_t*>(hp->x_host) + off_b, bytes, cudaMemcpyHostToDevice,
                          hp->h2d) != cudaSuccess ||
          cudaEventRecord(hp->ev[2 + k], hp->h2d) != cudaSuccess)
        return GDLA_ERR_CUDA;
    }
    for (int k = 0; k < hp->n_pieces; ++k) {
      const long long r0 = k * piece, r1 = r0 + piece < M ? r0 + piece : M;
      if (r0 >= r1) break;
      if (cudaStreamWaitEvent(st, hp->ev[2 + k], 0) != cudaSuccess) return GDLA_ERR_CUDA;
      if ((rc = down_proj_rows(cfg, w, x, D1, T, r0, r1, ctl, st))) return rc;
      if ((rc = norm_up_rows(cfg, w, ws, off, T, r0, r1, rope, err, ctl, st))) return rc;
    }
  } else {
    if ((rc = down_proj_rows(cfg, w, x, D1, T, 0, M, ctl, st))) return rc;
  }

  const int nqq = nH * (cfg->d_nope + cfg->d_rope);
  stage(1, st);
  if (!hp) {
  // a2: norms, rotary key, lambda, latent rows
  NormParams np{};
  np.D1 = D1; np.ld1 = ld1; np.M = M; np.q_rank = cfg->q_rank; np.kv_rank = cfg->kv_rank;
  np.n_signal = cfg->n_signal; np.g_q = w->g_q; np.g_kv = w->g_kv; np.eps = cfg->rms_eps;
  np.cQ = cQ; np.latent = latent; np.kR16 = kR16; np.lam = lam; np.pos_T = T; np.pos_ptr = positions;
  np.cache = kv_cache_out; np.cache_cap = cache_cap; np.rope = rope; np.err = err;
  if (ctx) {
    // local rows follow the prefix rows in the key-side buffers; positions continue the prefix
    np.pos_off = ctx->pos_offset;
    np.latent = static_cast<__nv_bfloat16*>(latent) + (size_t)n_pre * row_w;
    np.kR16 = static_cast<__half*>(kR16) + (size_t)n_pre * cfg->d_rope;
    if (latent_only) { np.latent = ctx->latent_out; np.kR16 = nullptr; }
    if (!latent_only && n_pre > 0) {
      if (cudaMemcpyAsync(latent, ctx->prefix_latent, (size_t)n_pre * row_w * 2,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return GDLA_ERR_CUDA;
      if (launch_failed(launch_latent_to_kr16(ctx->prefix_latent, cfg->kv_rank, n_pre, kR16, err, st)))
        return GDLA_ERR_LAUNCH;
    }
  }
  if (launch_failed(launch_norm_rope(np, st))) return GDLA_ERR_LAUNCH;
  if (latent_only) {
    stage(5, st);
    return GDLA_OK;
  }
  if (ctx && ctx->latent_out &&
      cudaMemcpyAsync(ctx->latent_out, static_cast<const __nv_bfloat16*>(latent) + (size_t)n_pre * row_w,
                      (size_t)M * row_w * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return GDLA_ERR_CUDA;

  stage(2, st);
  // a3: up-projections (q^C | rotated q^R), gate logits, K^C | V
  GemmEpi eq{};
  eq.C = QQ; eq.ldc = nqq; eq.out_type = OUT_F16; eq.M = M; eq.N = nqq;
  eq.rope_lo = nH * cfg->d_nope; eq.rope_hi = nqq; eq.pos_T = T; eq.pos_ptr = positions;
  eq.pos_off = ctx ? ctx->pos_offset : 0; eq.rope = rope;
  if (launch_failed(launch_gemm(cQ, cfg->q_rank, w->W_bQ, nqq, false, M, nqq, cfg->q_rank, eq, ctl, st)))
    return GDLA_ERR_LAUNCH;
  GemmEpi eg{};
  eg.C = G; eg.ldc = cfg->n_signal * cfg->d_v; eg.out_type = OUT_BF16; eg.M = M; eg.N = eg.ldc;
  eg.pos_T = T;
  if (launch_failed(launch_gemm(cQ, cfg->q_rank, w->W_G, eg.N, false, M, eg.N, cfg->q_rank, eg, ctl, st)))
    return GDLA_ERR_LAUNCH;
  GemmEpi ekv{};
  const int nkv = cfg->n_kv_heads * (cfg->d_nope + cfg->d_v);
  ekv.C = KV; ekv.ldc = nkv; ekv.out_type = OUT_F16; ekv.M = M + n_pre; ekv.N = nkv; ekv.pos_T = T;
  if (launch_failed(launch_gemm(latent, cfg->kv_rank + cfg->d_rope, w->W_bKV, nkv, false, M + n_pre, nkv,
                  cfg->kv_rank, ekv, ctl, st)))
    return GDLA_ERR_LAUNCH;
  }  // !hp (the host-buffer path ran a2 and a3 piece by piece above)

  stage(3, st);
  // a4: fused attention + differential combine + gate
  AttnParams ap{};
  ap.B = B; ap.T = T; ap.T_kv = T + n_pre; ap.q_off = n_pre; ap.window = cfg->window;
  ap.n_groups = cfg->n_noise;
  ap.n_signal = cfg->n_signal; ap.rope_col0 = nH * cfg->d_nope;
  ap.scale_log2 = float(1.4426950408889634 / sqrt(double(cfg->d_nope + cfg->d_rope)));
  ap.lam = lam; ap.G = G; ap.O_noise = On; ap.Dg = Dg;
  ap.units = units; ap.n_units = n_units; ap.max_units = max_units;
  if (launch_failed(launch_attn_prefill(QQ, nqq, KV, kR16, ap, ctl, st))) return GDLA_ERR_LAUNCH;

  stage(4, st);
  // a5: output projection (with host buffers: piece by piece, each piece of y leaving at once)
  if (hp) {
    const long long piece = (M + hp->n_pieces - 1) / hp->n_pieces;
    for (int k = 0; k < hp->n_pieces; ++k) {
      const long long r0 = k * piece, r1 = r0 + piece < M ? r0 + piece : M;
      if (r0 >= r1) break;
      if ((rc = out_proj_rows(cfg, w, Dg, y, T, r0, r1, ctl, st))) return rc;
      const size_t bytes = size_t(r1 - r0) * cfg->d_model * 2, off_b = size_t(r0) * cfg->d_model * 2;
      if (cudaEventRecord(hp->ev[2 + hp->n_pieces + k], st) != cudaSuccess ||
          cudaStreamWaitEvent(hp->d2h, hp->ev[2 + hp->n_pieces + k], 0) != cudaSuccess ||
          cudaMemcpyAsync(static_cast<uint8_t*>(hp->y_host) + off_b, static_cast<const uint8_t*>(y) + off_b,
                          bytes, cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess)
        return GDLA_ERR_CUDA;
    }
    // the caller's stream completes only after the last piece of y has reached the host
    if (cudaEventRecord(hp->ev[1], hp->d2h) != cudaSuccess || cudaStreamWaitEvent(st, hp->ev[1], 0) != cudaSuccess)
      return GDLA_ERR_CUDA;
  } else {
    if ((rc = out_proj_rows(cfg, w, Dg, y, T, 0, M, ctl, st))) return rc;
  }
  stage(5, st);
  return GDLA_OK;
}

}  // namespace gdla

using namespace gdla;

extern "C" {

const char* gdla_status_string(int s) {
  switch (s) {
    case GDLA_OK: return "ok";
    case GDLA_ERR_INVALID_ARG: return "invalid argument";
    case GDLA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case GDLA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case GDLA_ERR_LAUNCH: return "kernel launch failed";
    case GDLA_ERR_DEVICE_TIMEOUT: return "bounded in-kernel wait expired";
    case GDLA_ERR_CUDA: return "CUDA runtime error";
    case GDLA_ERR_DEVICE_DATA: return "a kernel met bad input data (see gdla_device_error)";
    default: return "unknown status";
  }
}

int gdla_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns = ns < 1000ull ? 1000ull : ns;
  return GDLA_OK;
}

// Host-buffer prefill: the prefill layout, then device copies of x and y.
static size_t host_extra_offset(const gdla_config_t* c, int B, int T, size_t* y_off, size_t* total) {
  size_t off[WS_N + 1];
  layout(c, B, T, GDLA_MODE_PREFILL, off);
  const size_t xy = ((size_t)B * T * c->d_model * 2 + 255) & ~size_t(255);
  *y_off = off[WS_N] + xy;
  *total = off[WS_N] + 2 * xy;
  return off[WS_N];
}

int gdla_workspace_size(const gdla_config_t* cfg, int B, int T, int mode, size_t* bytes) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!bytes || B <= 0 || (mode != GDLA_MODE_DECODE && T <= 0) ||
      (mode != GDLA_MODE_PREFILL && mode != GDLA_MODE_DECODE && mode != GDLA_MODE_VARLEN &&
       mode != GDLA_MODE_CONTEXT && mode != GDLA_MODE_HOST))
    return GDLA_ERR_INVALID_ARG;
  if (mode == GDLA_MODE_HOST) {
    size_t y_off;
    host_extra_offset(cfg, B, T, &y_off, bytes);
    return GDLA_OK;
  }
  size_t off[WS_N + 1];
  layout(cfg, B, T, mode, off);
  *bytes = off[WS_N];
  return GDLA_OK;
}

int gdla_workspace_offset(const gdla_config_t* cfg, int B, int T, int mode, int which,
                          size_t* offset) {
  size_t total;
  int rc = gdla_workspace_size(cfg, B, T, mode, &total);
  if (rc) return rc;
  if (!offset || which < 0 || which >= WS_N) return GDLA_ERR_INVALID_ARG;
  size_t off[WS_N + 1];
  layout(cfg, B, T, mode, off);
  *offset = off[which];
  return GDLA_OK;
}

// The absorbed tensors, in order: W_UKt, W_a, W_bqg (each rounded up to 256 bytes).
static void absorbed_layout(const gdla_config_t* c, size_t off[4]) {
  const int nH = c->n_signal + c->n_noise;
  const size_t sz[3] = {(size_t)c->n_kv_heads * c->d_nope * c->kv_rank * 2,
                        (size_t)c->d_model * (c->q_rank + c->kv_rank + c->d_rope + c->n_signal) * 2,
                        (size_t)c->q_rank * ((size_t)nH * (c->d_nope + c->d_rope) + (size_t)c->n_signal * c->d_v) * 2};
  size_t o = 0;
  for (int i = 0; i < 3; ++i) {
    off[i] = o;
    o += (sz[i] + 255) & ~size_t(255);
  }
  off[3] = o;
}

int gdla_absorbed_size(const gdla_config_t* cfg, size_t* bytes) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!bytes) return GDLA_ERR_INVALID_ARG;
  size_t off[4];
  absorbed_layout(cfg, off);
  *bytes = off[3];
  return GDLA_OK;
}

int gdla_prefill_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x, int B,
                     int T, void* y, void* kv_cache_out, int cache_cap, void* workspace,
                     size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_weights(w))) return rc;
  if (!x || !y || !workspace || B <= 0 || T <= 0) return GDLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return GDLA_ERR_INVALID_ARG;
  if ((long long)B * T > (1ll << 30)) return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (kv_cache_out && (cache_cap < T || !aligned16(kv_cache_out))) return GDLA_ERR_INVALID_ARG;
  size_t off[WS_N + 1];
  layout(cfg, B, T, GDLA_MODE_PREFILL, off);
  if (ws_bytes < off[WS_N]) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  return prefill_impl(cfg, w, x, B, T, y, kv_cache_out, cache_cap, static_cast<uint8_t*>(workspace),
                      off, static_cast<cudaStream_t>(stream), nullptr);
}

int gdla_prefill_varlen_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x,
                            int total, const int* cu_seqlens, int n_docs, void* y,
                            void* kv_latent_out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_weights(w))) return rc;
  if (!x || !y || !workspace || !cu_seqlens || total <= 0 || n_docs <= 0)
    return GDLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace) ||
      (kv_latent_out && !aligned16(kv_latent_out)))
    return GDLA_ERR_INVALID_ARG;
  if ((long long)total > (1ll << 30) || n_docs > total) return GDLA_ERR_UNSUPPORTED_SHAPE;
  size_t off[WS_N + 1];
  layout(cfg, 1, total, GDLA_MODE_VARLEN, off);
  if (ws_bytes < off[WS_N]) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  VarlenArgs vl{cu_seqlens, n_docs, kv_latent_out};
  return prefill_impl(cfg, w, x, 1, total, y, nullptr, 0, static_cast<uint8_t*>(workspace), off,
                      static_cast<cudaStream_t>(stream), &vl);
}

static int check_fp8_rows(const gdla_config_t* cfg, const void* a, long long rows, const void* b) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (cfg->kv_rank + cfg->d_rope != 576) return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (!a || !b || rows < 0 || !aligned16(a) || !aligned16(b)) return GDLA_ERR_INVALID_ARG;
  return GDLA_OK;
}

int gdla_quantize_latent_fp8(const gdla_config_t* cfg, const void* latent, long long rows, void* out,
                             void* stream) {
  int rc = check_fp8_rows(cfg, latent, rows, out);
  if (rc) return rc;
  return launch_failed(launch_mxfp8_quantize(latent, rows, out, static_cast<cudaStream_t>(stream)))
             ? GDLA_ERR_LAUNCH
             : GDLA_OK;
}

int gdla_dequantize_latent_fp8(const gdla_config_t* cfg, const void* stored, long long rows, void* out,
                               void* stream) {
  int rc = check_fp8_rows(cfg, stored, rows, out);
  if (rc) return rc;
  return launch_failed(launch_mxfp8_dequantize(stored, rows, out, static_cast<cudaStream_t>(stream)))
             ? GDLA_ERR_LAUNCH
             : GDLA_OK;
}

int gdla_latent_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x, int T,
                    int pos_offset, void* latent_out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_weights(w))) return rc;
  if (!x || !latent_out || !workspace || T <= 0 || pos_offset < 0) return GDLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(latent_out) || !aligned16(workspace)) return GDLA_ERR_INVALID_ARG;
  if ((long long)T + pos_offset > (1ll << 30)) return GDLA_ERR_UNSUPPORTED_SHAPE;
  size_t off[WS_N + 1];
  layout(cfg, 1, T, GDLA_MODE_PREFILL, off);
  if (ws_bytes < off[WS_N]) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  ContextArgs ctx{nullptr, 0, pos_offset, latent_out};
  return prefill_impl(cfg, w, x, 1, T, nullptr, nullptr, 0, static_cast<uint8_t*>(workspace), off,
                      static_cast<cudaStream_t>(stream), nullptr, &ctx, true);
}

int gdla_prefill_context_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x, int T,
                             int pos_offset, const void* prefix_latent, int n_prefix, void* y,
                             void* latent_out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_weights(w))) return rc;
  if (!x || !y || !workspace || T <= 0 || n_prefix < 0 || pos_offset < n_prefix ||
      (n_prefix > 0 && !prefix_latent))
    return GDLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace) ||
      (prefix_latent && !aligned16(prefix_latent)) || (latent_out && !aligned16(latent_out)))
    return GDLA_ERR_INVALID_ARG;
  if ((long long)T + pos_offset > (1ll << 30)) return GDLA_ERR_UNSUPPORTED_SHAPE;
  size_t off[WS_N + 1];
  layout(cfg, 1, T + n_prefix, GDLA_MODE_CONTEXT, off);
  if (ws_bytes < off[WS_N]) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  ContextArgs ctx{prefix_latent, n_prefix, pos_offset, latent_out};
  return prefill_impl(cfg, w, x, 1, T, y, nullptr, 0, static_cast<uint8_t*>(workspace), off,
                      static_cast<cudaStream_t>(stream), nullptr, &ctx, false);
}

// Copy streams and events of the host-buffer prefill, one set per device, created on first use
// and kept for the life of the process (like the device error word).
namespace {
constexpr int kMaxPieces = 64;
struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev[2 * kMaxPieces + 2];
};
constexpr int kMaxDevices = 64;
HostPipe g_pipes[kMaxDevices];
std::mutex g_pipe_mu;
}  // namespace

static int host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& p = g_pipes[dev];
  if (!p.ready) {
    if (cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking) != cudaSuccess)
      return GDLA_ERR_CUDA;
    for (auto& e : p.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return GDLA_ERR_CUDA;
    p.ready = true;
  }
  *out = &p;
  return GDLA_OK;
}

int gdla_prefill_host_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x_host, int B,
                          int T, void* y_host, int n_pieces, void* workspace, size_t ws_bytes,
                          void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_weights(w))) return rc;
  if (!x_host || !y_host || !workspace || B <= 0 || T <= 0 || n_pieces < 1 || n_pieces > kMaxPieces)
    return GDLA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return GDLA_ERR_INVALID_ARG;
  if ((long long)B * T > (1ll << 30)) return GDLA_ERR_UNSUPPORTED_SHAPE;
  size_t y_off, total;
  const size_t x_off = host_extra_offset(cfg, B, T, &y_off, &total);
  if (ws_bytes < total) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  HostPipe* pipe;
  if ((rc = host_pipe(&pipe))) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t off[WS_N + 1];
  layout(cfg, B, T, GDLA_MODE_PREFILL, off);
  HostPipeArgs hp{x_host, y_host, n_pieces, pipe->h2d, pipe->d2h, pipe->ev};
  return prefill_impl(cfg, w, ws + x_off, B, T, ws + y_off, nullptr, 0, ws, off,
                      static_cast<cudaStream_t>(stream), nullptr, nullptr, false, &hp);
}

// ---------------------------------------------------------------- attention stage for training
int gdla_attn_train_workspace_size(const gdla_config_t* cfg, int B, int T, size_t* fwd_bytes,
                                   size_t* bwd_bytes) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!fwd_bytes || !bwd_bytes || B <= 0 || T <= 0) return GDLA_ERR_INVALID_ARG;
  const long long M = (long long)B * T;
  *fwd_bytes = (size_t)((M + 31) / 32 * 32) * cfg->n_noise * cfg->d_v * 4;
  *bwd_bytes = attn_bwd_workspace_bytes(M, T, cfg->n_signal + cfg->n_noise, cfg->n_noise);
  return GDLA_OK;
}

int gdla_attn_train_fwd(const gdla_config_t* cfg, const void* qq, const void* kv, const void* kr16,
                        const float* lam, const void* gate, int B, int T, void* dg_out, void* h_out,
                        float* lse_out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!qq || !kv || !kr16 || !lam || !gate || !dg_out || !h_out || !lse_out || !workspace || B <= 0 || T <= 0)
    return GDLA_ERR_INVALID_ARG;
  for (const void* ptr : {qq, kv, kr16, (const void*)lam, gate, (const void*)dg_out, (const void*)h_out,
                          (const void*)lse_out, (const void*)workspace})
    if (!aligned16(ptr)) return GDLA_ERR_INVALID_ARG;
  if ((long long)B * T > (1ll << 30)) return GDLA_ERR_UNSUPPORTED_SHAPE;
  size_t fb, bb;
  gdla_attn_train_workspace_size(cfg, B, T, &fb, &bb);
  if (ws_bytes < fb) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  int* err;
  if ((rc = error_word(&err))) return rc;
  KernelCtlHost ctl{err, g_wait_limit_ns};
  const int nH = cfg->n_signal + cfg->n_noise;
  AttnParams ap{};
  ap.B = B; ap.T = T; ap.T_kv = T; ap.q_off = 0; ap.window = cfg->window; ap.n_groups = cfg->n_noise;
  ap.n_signal = cfg->n_signal; ap.rope_col0 = nH * cfg->d_nope;
  ap.scale_log2 = float(1.4426950408889634 / sqrt(double(cfg->d_nope + cfg->d_rope)));
  ap.lam = lam; ap.G = gate; ap.O_noise = static_cast<float*>(workspace); ap.Dg = dg_out;
  ap.H_out = h_out; ap.lse_out = lse_out;
  if (launch_failed(launch_attn_prefill(qq, nH * (cfg->d_nope + cfg->d_rope), kv, kr16, ap, ctl,
                                        static_cast<cudaStream_t>(stream))))
    return GDLA_ERR_LAUNCH;
  return GDLA_OK;
}

int gdla_attn_bwd(const gdla_config_t* cfg, const void* qq, const void* kv, const void* kr16,
                  const float* lam, const void* gate, const void* h, const float* lse, const void* d_dg,
                  int B, int T, float* d_qq, float* d_kv, float* d_kr, float* d_lam, float* d_gate,
                  void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  for (const void* ptr : {qq, kv, kr16, (const void*)lam, gate, h, (const void*)lse, d_dg, (const void*)d_qq,
                          (const void*)d_kv, (const void*)d_kr, (const void*)d_lam, (const void*)d_gate,
                          (const void*)workspace})
    if (!ptr || !aligned16(ptr)) return GDLA_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0) return GDLA_ERR_INVALID_ARG;
  if ((long long)B * T > (1ll << 30)) return GDLA_ERR_UNSUPPORTED_SHAPE;
  size_t fb, bb;
  gdla_attn_train_workspace_size(cfg, B, T, &fb, &bb);
  if (ws_bytes < bb) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  AttnBwdParams a{};
  a.B = B; a.T = T; a.window = cfg->window; a.n_signal = cfg->n_signal; a.n_groups = cfg->n_noise;
  a.scale = float(1.0 / sqrt(double(cfg->d_nope + cfg->d_rope)));
  a.scale_log2 = float(1.4426950408889634 / sqrt(double(cfg->d_nope + cfg->d_rope)));
  a.QQ = qq; a.KV = kv; a.kR16 = kr16; a.lam = lam; a.G = gate; a.H = h; a.lse = lse; a.d_dg = d_dg;
  a.d_qq = d_qq; a.d_kv = d_kv; a.d_kr = d_kr; a.d_lam = d_lam; a.d_G = d_gate; a.ws = workspace;
  int* err;
  if ((rc = error_word(&err))) return rc;
  KernelCtlHost ctl{err, g_wait_limit_ns};
  rc = launch_attn_bwd(a, ctl, static_cast<cudaStream_t>(stream));
  if (rc == 0) {
    g_launches += 6;   // pre-pass, two gathers, dK/dV, dq, dk^R reduce
    return GDLA_OK;
  }
  return GDLA_ERR_LAUNCH;
}

int gdla_absorb_weights(const gdla_config_t* cfg, const gdla_weights_t* w, void* dst,
                        size_t dst_bytes, gdla_absorbed_t* out, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_weights(w))) return rc;
  if (!dst || !out || !aligned16(dst)) return GDLA_ERR_INVALID_ARG;
  size_t need;
  gdla_absorbed_size(cfg, &need);
  if (dst_bytes < need) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  size_t off[4];
  absorbed_layout(cfg, off);
  uint8_t* base = static_cast<uint8_t*>(dst);
  if (launch_failed(launch_absorb_uk(w->W_bKV, base + off[0], cfg->kv_rank, cfg->n_kv_heads, cfg->d_nope,
                                     cfg->d_v, st)))
    return GDLA_ERR_LAUNCH;
  // W_a = [W_a^Q | W_a^KV | W^lambda] and W_bqg = [W_b^Q | W^G], so that each of the two
  // products of the query path is one GEMM
  const int nH = cfg->n_signal + cfg->n_noise;
  const long long lda = cfg->q_rank + cfg->kv_rank + cfg->d_rope + cfg->n_signal;
  const long long nqq = (long long)nH * (cfg->d_nope + cfg->d_rope);
  const long long ldb = nqq + (long long)cfg->n_signal * cfg->d_v;
  const int nkv = cfg->kv_rank + cfg->d_rope;
  if (launch_failed(launch_copy_cols(w->W_aQ, cfg->q_rank, base + off[1], lda, 0, cfg->d_model, cfg->q_rank, st)) ||
      launch_failed(launch_copy_cols(w->W_aKV, nkv, base + off[1], lda, cfg->q_rank, cfg->d_model, nkv, st)) ||
      launch_failed(launch_copy_cols(w->W_lambda, cfg->n_signal, base + off[1], lda, cfg->q_rank + nkv,
                                     cfg->d_model, cfg->n_signal, st)) ||
      launch_failed(launch_copy_cols(w->W_bQ, nqq, base + off[2], ldb, 0, cfg->q_rank, int(nqq), st)) ||
      launch_failed(launch_copy_cols(w->W_G, (long long)cfg->n_signal * cfg->d_v, base + off[2], ldb, int(nqq),
                                     cfg->q_rank, cfg->n_signal * cfg->d_v, st)))
    return GDLA_ERR_LAUNCH;
  out->w = *w;
  out->W_UKt = base + off[0];
  out->W_a = base + off[1];
  out->W_bqg = base + off[2];
  out->cfg = *cfg;
  out->magic = kAbsorbedMagic;
  return GDLA_OK;
}

int gdla_decode_fwd(const gdla_config_t* cfg, const gdla_absorbed_t* ab, const void* x_new,
                    void* kv_cache, const int* cache_len, int cap, int B, void* y, void* workspace,
                    size_t ws_bytes, void* stream) {
  return gdla_decode_multi_fwd(cfg, ab, x_new, 1, kv_cache, cache_len, cap, B, y, workspace,
                               ws_bytes, stream);
}

// The decode step over a bf16 latent cache or an MXFP8 one (fp8): the same kernels, except
// that the new rows are appended in MXFP8 form and the attention converts the cache tiles.
static int decode_impl(const gdla_config_t* cfg, const gdla_absorbed_t* ab, const void* x_new, int q_len,
                       void* kv_cache, const int* cache_len, int cap, int n_seq, void* y, void* workspace,
                       size_t ws_bytes, void* stream, bool fp8) {
  if (q_len <= 0 || n_seq <= 0 || (long long)q_len * n_seq > (1 << 20)) return GDLA_ERR_INVALID_ARG;
  const int B = q_len * n_seq;   // query rows: token r % q_len of sequence r / q_len
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!ab || ab->magic != kAbsorbedMagic || !ab->W_UKt || !ab->W_a || !ab->W_bqg) return GDLA_ERR_INVALID_ARG;
  if (ab->cfg.d_model != cfg->d_model || ab->cfg.n_noise != cfg->n_noise)
    return GDLA_ERR_INVALID_ARG;  // absorbed for another layer shape (the window may differ)
  const gdla_weights_t* w = &ab->w;
  if ((rc = check_weights(w))) return rc;
  if (!x_new || !kv_cache || !cache_len || !y || !workspace || B <= 0 || cap <= 0)
    return GDLA_ERR_INVALID_ARG;
  if (!aligned16(x_new) || !aligned16(kv_cache) || !aligned16(y) || !aligned16(workspace))
    return GDLA_ERR_INVALID_ARG;
  size_t off[WS_N + 1];
  layout(cfg, B, cap, GDLA_MODE_DECODE, off);
  if (ws_bytes < off[WS_N]) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err;
  if ((rc = error_word(&err))) return rc;
  KernelCtlHost ctl{err, g_wait_limit_ns};
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* D1 = reinterpret_cast<float*>(ws + off[WS_D1]);
  void* cQ = ws + off[WS_CQ];
  float* lam = reinterpret_cast<float*>(ws + off[WS_LAM]);
  float* QQ = reinterpret_cast<float*>(ws + off[WS_QQ]);
  void* qt = ws + off[WS_KV];
  float* part = reinterpret_cast<float*>(ws + off[WS_ONOISE]);
  float* ml = reinterpret_cast<float*>(ws + off[WS_KR16]);
  void* Dg = ws + off[WS_DG];
  const int nH = cfg->n_signal + cfg->n_noise;
  const int ld1 = cfg->q_rank + cfg->kv_rank + cfg->d_rope + cfg->n_signal;
  RopeTable rope;
  fill_rope_table(&rope, cfg->d_rope, cfg->rope_theta);

  stage(0, st);
  float* splitk = reinterpret_cast<float*>(ws + off[WS_SPLITK]);
  const long long splitk_n = decode_splitk_floats(cfg, B);
  GemmEpi ep{};
  ep.ldc = ld1; ep.out_type = OUT_F32; ep.M = B; ep.pos_T = 1; ep.rope = rope;
  ep.splitk = splitk; ep.splitk_floats = splitk_n;
  // [c^Q | c^KV | k^R | lambda logits] = x [W_a^Q | W_a^KV | W^lambda]: one product
  ep.C = D1; ep.N = ld1;
  if (launch_failed(launch_gemm(x_new, cfg->d_model, ab->W_a, ld1, false, B, ld1, cfg->d_model, ep, ctl, st)))
    return GDLA_ERR_LAUNCH;

  NormParams np{};
  np.D1 = D1; np.ld1 = ld1; np.M = B; np.q_rank = cfg->q_rank; np.kv_rank = cfg->kv_rank;
  np.n_signal = cfg->n_signal; np.g_q = w->g_q; np.g_kv = w->g_kv; np.eps = cfg->rms_eps;
  np.cQ = cQ; np.latent = nullptr; np.kR16 = nullptr; np.lam = lam; np.pos_T = 1;
  np.pos_ptr = cache_len; np.q_per_seq = q_len; np.cache = kv_cache; np.cache_fp8 = fp8; np.cache_cap = cap;
  np.rope = rope; np.err = err;
  if (launch_failed(launch_norm_rope(np, st))) return GDLA_ERR_LAUNCH;

  // [q^C | q^R (rotated at the token's position) | G] = c^Q [W_b^Q | W^G], fp32: one product
  const int nqq = nH * (cfg->d_nope + cfg->d_rope);
  const int ldq = nqq + cfg->n_signal * cfg->d_v;
  GemmEpi eq{};
  eq.C = QQ; eq.ldc = ldq; eq.out_type = OUT_F32; eq.M = B; eq.N = ldq;
  eq.rope_lo = nH * cfg->d_nope; eq.rope_hi = nqq; eq.pos_T = 1; eq.pos_ptr = cache_len;
  eq.pos_div = q_len;
  eq.rope = rope; eq.splitk = splitk; eq.splitk_floats = splitk_n;
  if (launch_failed(launch_gemm(cQ, cfg->q_rank, ab->W_bqg, ldq, false, B, ldq, cfg->q_rank, eq, ctl, st)))
    return GDLA_ERR_LAUNCH;

  DecQParams qp{};
  qp.B = B; qp.n_groups = cfg->n_noise; qp.n_signal = cfg->n_signal; qp.n_heads = nH;
  qp.QQ = QQ; qp.qq_ld = ldq; qp.rope_col0 = nH * cfg->d_nope; qp.W_UKt = ab->W_UKt; qp.qt = qt;
  qp.qt_f16 = fp8;
  if (launch_failed(launch_qtilde(qp, ctl, st))) return GDLA_ERR_LAUNCH;

  DecAttnParams dp{};
  dp.R = B; dp.n_seq = n_seq; dp.cap = cap; dp.window = cfg->window; dp.cache_len = cache_len;
  dp.q_len = q_len;
  dp.cache = kv_cache; dp.cache_fp8 = fp8; dp.qt = qt;
  dp.scale_log2 = float(1.4426950408889634 / sqrt(double(cfg->d_nope + cfg->d_rope)));
  dp.tstart = reinterpret_cast<int*>(ws + off[WS_DSCHED]);
  dp.n_ctas = decode_cta_count();
  dp.part = part; dp.ml = ml; dp.err = err;
  if (nH != 80) return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (launch_failed(launch_dec_sched(dp, st))) return GDLA_ERR_LAUNCH;

  stage(1, st);
  if (launch_failed(launch_dec_attn_tc(dp, ctl, st))) return GDLA_ERR_LAUNCH;

  stage(2, st);
  DecCombParams cp{};
  cp.B = B; cp.n_groups = cfg->n_noise; cp.n_signal = cfg->n_signal; cp.n_ctas = dp.n_ctas;
  cp.q_len = q_len; cp.n_seq = n_seq;
  cp.tstart = dp.tstart;
  cp.part = part; cp.ml = ml; cp.lam = lam; cp.G = QQ + nqq; cp.g_ld = ldq; cp.W_bKV = w->W_bKV; cp.Dg = Dg;
  if (launch_failed(launch_dec_combine(cp, ctl, st))) return GDLA_ERR_LAUNCH;

  stage(3, st);
  GemmEpi eo{};
  eo.C = y; eo.ldc = cfg->d_model; eo.out_type = OUT_BF16; eo.M = B; eo.N = cfg->d_model;
  eo.pos_T = 1; eo.splitk = splitk; eo.splitk_floats = splitk_n;
  if (launch_failed(launch_gemm(Dg, cfg->n_signal * cfg->d_v, w->W_O, cfg->d_model, false, B, cfg->d_model,
                  cfg->n_signal * cfg->d_v, eo, ctl, st)))
    return GDLA_ERR_LAUNCH;
  stage(4, st);
  return GDLA_OK;
}

int gdla_decode_multi_fwd(const gdla_config_t* cfg, const gdla_absorbed_t* ab, const void* x_new,
                          int q_len, void* kv_cache, const int* cache_len, int cap, int n_seq,
                          void* y, void* workspace, size_t ws_bytes, void* stream) {
  return decode_impl(cfg, ab, x_new, q_len, kv_cache, cache_len, cap, n_seq, y, workspace, ws_bytes, stream,
                     false);
}

int gdla_decode_fp8_fwd(const gdla_config_t* cfg, const gdla_absorbed_t* ab, const void* x_new, int q_len,
                        void* kv_cache8, const int* cache_len, int cap, int n_seq, void* y, void* workspace,
                        size_t ws_bytes, void* stream) {
  if (cfg && cfg->kv_rank + cfg->d_rope != 576) return GDLA_ERR_UNSUPPORTED_SHAPE;
  return decode_impl(cfg, ab, x_new, q_len, kv_cache8, cache_len, cap, n_seq, y, workspace, ws_bytes, stream,
                     true);
}

int gdla_set_stage_events(void* const* events, int n) {
  if (n < 0 || n > 8 || (n > 0 && !events)) return GDLA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!events[i]) return GDLA_ERR_INVALID_ARG;
    g_stage_ev[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_n_stage_ev = n;
  return GDLA_OK;
}

unsigned long long gdla_kernel_launches(void) { return g_launches; }

int gdla_device_error(void* stream, int* site, int clear) {
  if (!site) return GDLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return GDLA_ERR_CUDA;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return GDLA_ERR_CUDA;
  }
  *site = v;
  if (!v) return GDLA_OK;
  // 0x6xx / 0x7xx: a kernel met bad input data; the other sites are expired waits
  return (v >= 0x600 && v < 0x800) ? GDLA_ERR_DEVICE_DATA : GDLA_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"

namespace gdla {
// One CTA waits on an mbarrier that nothing ever arrives on: the bounded wait must expire,
// record its site code and return, and the kernel must then exit normally.
__global__ void selftest_wait_kernel(KernelCtl ctl) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ctl, SITE_SELFTEST);
}
}  // namespace gdla

extern "C" int gdla_selftest_wait_timeout(unsigned long long limit_ns, void* stream, int* site) {
  if (!site) return GDLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err;
  int rc = error_word(&err);
  if (rc) return rc;
  KernelCtl kc{err, limit_ns < 1000ull ? 1000ull : limit_ns};
  int prev = 0;
  if (cudaMemcpyFromSymbol(&prev, g_device_error, sizeof(int)) != cudaSuccess) return GDLA_ERR_CUDA;
  if (prev) return GDLA_ERR_DEVICE_TIMEOUT;  // an earlier failure is still unread
  selftest_wait_kernel<<<1, 32, 0, st>>>(kc);
  if (cudaPeekAtLastError() != cudaSuccess) return GDLA_ERR_LAUNCH;
  ++g_launches;
  return gdla_device_error(stream, site, 1);
}
