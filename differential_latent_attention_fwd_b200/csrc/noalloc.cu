// Allocation-free entry point for the fused prefill attention stage.
//
// Some callers cannot allocate device memory at the time they run GDLA: for example a plugin
// inside an inference engine that owns every device buffer and hands the plugin only its
// inputs and outputs, or a service that forbids allocations after start-up so that its memory
// footprint stays fixed.  gdla_prefill_fwd needs a caller-provided workspace; this entry point
// instead keeps the only scratch the attention stage needs (the normalised noise-head outputs
// that the signal heads subtract) in a fixed array compiled into the library.
//
// The array lives in device memory for as long as the library is loaded, on every GPU that
// loads it: GDLA_NOALLOC_MAX_TOKENS tokens x 16 noise heads x 128 values x 4 bytes = 32 MiB.
#include "../../include/gdla.h"
#include "gdla_common.cuh"
#include "gdla_internal.h"

#include <mutex>

namespace gdla {

namespace {
constexpr int kMaxNoise = 16;
constexpr size_t kScratchFloats = size_t(GDLA_NOALLOC_MAX_TOKENS) * kMaxNoise * 128;

// Noise-head outputs of the current call.  Every element a call reads is written earlier in
// the same call, so nothing needs clearing; calls that overlap on the GPU share it and race.
static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Per device: the context the address was looked up in, and the address.  A device reset (or
// any teardown of the primary context) gives the device a new context with a new ID, and the
// next call looks the address up again instead of using a pointer into the old context.
unsigned long long g_scratch_ctx[kMaxDevices] = {};
float* g_scratch_ptr[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique ID (for the process's life) of the calling thread's current context; 0 if unknown.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked = false;
  if (!looked) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  It is looked up once per device
// (and again after the device's context was recreated), with that device current.  In host code
// g_noalloc_scratch names a host-side shadow, never the device memory itself.
int scratch_on_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDLA_ERR_CUDA;
  // (no current context yet: ID 0, and the lookup below creates the device's primary context)
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDLA_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return GDLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

}  // namespace gdla

extern "C" int gdla_attn_prefill_noalloc(const gdla_config_t* cfg, const void* qq, const void* kv,
                                         const void* kr16, const float* lam, const void* gate,
                                         void* dg, int B, int T, void* stream) {
  using namespace gdla;
  if (!cfg || !qq || !kv || !kr16 || !lam || !gate || !dg || B <= 0 || T <= 0)
    return GDLA_ERR_INVALID_ARG;
  if (cfg->d_nope != 128 || cfg->d_rope != 64 || cfg->d_v != 128 || cfg->n_noise <= 0 ||
      cfg->n_noise > kMaxNoise || cfg->n_signal != 4 * cfg->n_noise || cfg->n_kv_heads != cfg->n_noise)
    return GDLA_ERR_UNSUPPORTED_SHAPE;
  if (cfg->window < 0) return GDLA_ERR_INVALID_ARG;
  if (!aligned16(qq) || !aligned16(kv) || !aligned16(kr16) || !aligned16(lam) || !aligned16(gate) ||
      !aligned16(dg))
    return GDLA_ERR_INVALID_ARG;
  if ((long long)B * T > GDLA_NOALLOC_MAX_TOKENS) return GDLA_ERR_WORKSPACE_TOO_SMALL;
  float* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc) return rc;
  KernelCtlHost ctl;
  if ((rc = shared_kernel_ctl(&ctl))) return rc;
  const int nH = cfg->n_signal + cfg->n_noise;
  AttnParams ap{};
  ap.B = B; ap.T = T; ap.T_kv = T; ap.q_off = 0; ap.window = cfg->window; ap.n_groups = cfg->n_noise;
  ap.n_signal = cfg->n_signal; ap.rope_col0 = nH * cfg->d_nope;
  ap.scale_log2 = float(1.4426950408889634 / sqrt(double(cfg->d_nope + cfg->d_rope)));
  ap.lam = lam; ap.G = gate; ap.O_noise = scratch; ap.Dg = dg;
  if (launch_attn_prefill(qq, nH * (cfg->d_nope + cfg->d_rope), kv, kr16, ap, ctl,
                          static_cast<cudaStream_t>(stream)))
    return GDLA_ERR_LAUNCH;
  return GDLA_OK;
}
