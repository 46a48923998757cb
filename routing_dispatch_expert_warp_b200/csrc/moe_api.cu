// The C ABI (include/moe.h): argument checks, workspace layout and the stage sequence.
// Host code only; every step of the layer runs in the kernels of the other files.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>

#include "moe_internal.h"

namespace moe {
namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_wait_ns{2000000000ull};

moe_status_t fail(moe_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

moe_status_t cuda_fail(cudaError_t err, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }

moe_status_t check_config(const moe_config_t* cfg, Shape* s) {
  if (cfg == nullptr) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->T < 1 || cfg->T > 2147483647LL)
    return fail(MOE_ERR_INVALID_ARG, "T must be in [1, 2^31) (got %lld)", (long long)cfg->T);
  if (cfg->d_model > (1LL << 24) || cfg->d_ff > (1LL << 24))
    return fail(MOE_ERR_INVALID_ARG, "d_model and d_ff must be at most 2^24");
  if (cfg->d_model < 8 || cfg->d_model % 8 != 0)
    return fail(MOE_ERR_INVALID_ARG, "d_model must be a positive multiple of 8 (got %lld)",
                (long long)cfg->d_model);
  if (cfg->d_ff < 4 || cfg->d_ff % 4 != 0)
    return fail(MOE_ERR_INVALID_ARG, "d_ff must be a positive multiple of 4 (got %lld)",
                (long long)cfg->d_ff);
  if (cfg->E < 1 || cfg->E > MOE_MAX_EXPERTS)
    return fail(MOE_ERR_INVALID_ARG, "E must be in [1, %d] (got %d)", MOE_MAX_EXPERTS, cfg->E);
  if (cfg->k < 1 || cfg->k > cfg->E || cfg->k > MOE_MAX_TOPK)
    return fail(MOE_ERR_INVALID_ARG, "k must be in [1, min(E, %d)] (got k=%d, E=%d)",
                MOE_MAX_TOPK, cfg->k, cfg->E);
  if (cfg->gating != MOE_GATE_SOFTMAX && cfg->gating != MOE_GATE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "unknown gating %d", cfg->gating);
  if (cfg->layout != MOE_LAYOUT_COMPACT && cfg->layout != MOE_LAYOUT_PADDED)
    return fail(MOE_ERR_INVALID_ARG, "unknown layout %d", cfg->layout);
  if (cfg->dtype != MOE_F32 && cfg->dtype != MOE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "unknown dtype %d", cfg->dtype);
  if (!(cfg->capacity_factor == cfg->capacity_factor))
    return fail(MOE_ERR_INVALID_ARG, "capacity_factor is NaN");
  if (cfg->n_groups > 1) {
    if (cfg->E % cfg->n_groups != 0)
      return fail(MOE_ERR_INVALID_ARG, "E (%d) must be a multiple of n_groups (%d)", cfg->E,
                  cfg->n_groups);
    if (cfg->topk_groups < 1 || cfg->topk_groups > cfg->n_groups ||
        static_cast<int64_t>(cfg->topk_groups) * (cfg->E / cfg->n_groups) < cfg->k)
      return fail(MOE_ERR_INVALID_ARG,
                  "topk_groups must be in [1, n_groups] and hold at least k experts");
  } else if (cfg->n_groups < 0) {
    return fail(MOE_ERR_INVALID_ARG, "n_groups must be >= 0");
  }
  if (cfg->bias_mode != MOE_BIAS_SCORE_AND_WEIGHT && cfg->bias_mode != MOE_BIAS_SELECTION_ONLY)
    return fail(MOE_ERR_INVALID_ARG, "unknown bias_mode %d", cfg->bias_mode);
  if (cfg->drop_policy != MOE_DROP_TOKEN_ORDER && cfg->drop_policy != MOE_DROP_PICK_RANK &&
      cfg->drop_policy != MOE_DROP_SCORE)
    return fail(MOE_ERR_INVALID_ARG, "unknown drop_policy %d", cfg->drop_policy);
  s->T = cfg->T;
  s->d = cfg->d_model;
  s->f = cfg->d_ff;
  s->E = cfg->E;
  s->k = cfg->k;
  s->gating = cfg->gating;
  s->layout = cfg->layout;
  s->dtype = cfg->dtype;
  s->n_groups = cfg->n_groups > 1 ? cfg->n_groups : 0;
  s->topk_groups = cfg->n_groups > 1 ? cfg->topk_groups : 0;
  s->bias_mode = cfg->bias_mode;
  s->drop_policy = cfg->drop_policy;
  s->elem = cfg->dtype == MOE_F32 ? 4 : 2;
  const int64_t A = cfg->T * cfg->k;
  if (cfg->capacity_factor > 0.0f) {
    const double c = ceil(static_cast<double>(cfg->capacity_factor) * static_cast<double>(cfg->T) *
                          static_cast<double>(cfg->k) / static_cast<double>(cfg->E));
    if (c > 2147483647.0) return fail(MOE_ERR_INVALID_ARG, "capacity too large");
    s->C = static_cast<int64_t>(c);
  } else {
    s->C = -1;
  }
  if (s->layout == MOE_LAYOUT_PADDED) {
    if (s->C < 0)
      return fail(MOE_ERR_INVALID_ARG, "PADDED layout needs capacity_factor > 0");
    s->max_rows = static_cast<int64_t>(s->E) * s->C;
  } else {
    s->max_rows = s->C < 0 ? A : (A < s->E * s->C ? A : s->E * s->C);
  }
  if (s->max_rows > 2147483647LL || A > 2147483647LL)
    return fail(MOE_ERR_INVALID_ARG, "too many rows for 32-bit row indices");
  if (cfg->dtype == MOE_F32 && cfg->d_ff % 4 != 0)
    return fail(MOE_ERR_INVALID_ARG, "fp32 d_ff must be a multiple of 4");
  return MOE_OK;
}

moe_status_t check_ws(const Shape& s, const void* ws, size_t ws_bytes, WsLayout* lay) {
  *lay = workspace_layout(s);
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0)
    return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < lay->total)
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, lay->total);
  return MOE_OK;
}

#define MOE_REQUIRE(cond, ...)                                 \
  do {                                                         \
    if (!(cond)) return fail(MOE_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

DevStatus* ws_status(void* ws, const WsLayout& lay) {
  return reinterpret_cast<DevStatus*>(static_cast<uint8_t*>(ws) + lay.status);
}

}  // namespace

WsLayout workspace_layout(const Shape& s) {
  WsLayout l;
  size_t off = 0;
  l.status = off;
  off += round_up(sizeof(DevStatus));
  l.hist = off;
  l.hist_bytes = round_up(dispatch_hist_bytes(s));
  off += l.hist_bytes;
  l.logits = off;
  l.logits_bytes = round_up(static_cast<size_t>(s.T) * s.E * sizeof(float));
  off += l.logits_bytes;
  const int splits = router_splits(s);
  l.partials = off;
  if (s.E <= 32) {  // lane-ordered copy of W_r for the small-E router
    const size_t et = s.E <= 8 ? 8 : (s.E <= 16 ? 16 : 32);
    l.partials_bytes = round_up(static_cast<size_t>((s.d + 255) / 256) * 256 * et * sizeof(float));
  } else {
    int kb_per = 0;
    const int parts = router_uses_tensor_cores(s) ? router_tc_splits(s, &kb_per) : splits;
    l.partials_bytes =
        parts > 1 ? round_up(static_cast<size_t>(parts) * s.T * s.E * sizeof(float)) : 0;
  }
  off += l.partials_bytes;
  l.router_tc = off;
  l.router_tc_bytes = round_up(router_tc_workspace_bytes(s));
  off += l.router_tc_bytes;
  l.ep_base = off;
  off += round_up(static_cast<size_t>(s.E) * sizeof(int32_t));
  l.arrive = off;
  off += round_up(static_cast<size_t>(s.T) * ((s.d + 255) / 256) * sizeof(int32_t));
  l.score = off;
  off += round_up(dispatch_score_scratch_bytes(s));
  l.total = off;
  return l;
}

int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// ------------------------------------------------------------------ bounded-wait self-test
namespace {
__global__ void wait_selftest_kernel(DevStatus* status, uint64_t wait_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    // nothing ever arrives on `bar`: the wait must run out and report, not hang
    if (!mbar_wait(&bar, 0, wait_ns, nullptr)) record_error(status, DEV_TIMEOUT, 99, 0);
  }
}
}  // namespace

namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

cudaError_t launch_wait_selftest(DevStatus* status, uint64_t wait_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, wait_ns);
  note_launch();
  return cudaGetLastError();
}

}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

uint64_t moe_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* moe_last_error(void) { return g_last_error.c_str(); }

const char* moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE_DATA: return "MOE_ERR_DEVICE_DATA";
  }
  return "unknown";
}

void moe_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns == 0 ? 2000000000ull : ns); }

moe_status_t moe_set_ffn_kernel(moe_ffn_kernel_t kind) {
  MOE_REQUIRE(kind == MOE_FFN_TOKEN_MAJOR || kind == MOE_FFN_CTA_PAIRS || kind == MOE_FFN_TOKEN_N,
              "moe_set_ffn_kernel: unknown kernel %d", static_cast<int>(kind));
  set_ffn_kernel(kind);
  return MOE_OK;
}


moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(bytes != nullptr, "bytes is NULL");
  *bytes = workspace_layout(s).total;
  return MOE_OK;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(ws != nullptr, "workspace is NULL");
  MOE_REQUIRE(ws_bytes >= sizeof(DevStatus), "workspace too small");
  cudaError_t err = cudaMemsetAsync(ws, 0, sizeof(DevStatus), static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_workspace_init");
  return MOE_OK;
}

int64_t moe_capacity(const moe_config_t* cfg) {
  Shape s;
  if (check_config(cfg, &s) != MOE_OK) return -2;
  return s.C;
}

int64_t moe_max_rows(const moe_config_t* cfg) {
  Shape s;
  if (check_config(cfg, &s) != MOE_OK) return -2;
  return s.max_rows;
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const float* w_router,
                       const float* logit_bias, int64_t bias_row_stride, float* logits,
                       int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                       void* stream) {
  return moe_route_ex(cfg, x, w_router, nullptr, logit_bias, bias_row_stride, logits, topk_idx,
                      topk_w, ws, ws_bytes, stream);
}

moe_status_t moe_router_split_size(const moe_config_t* cfg, size_t* bytes) {
  MOE_REQUIRE(bytes != nullptr, "moe_router_split_size: bytes is NULL");
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  *bytes = router_split_bytes(s);
  return MOE_OK;
}

moe_status_t moe_router_split(const moe_config_t* cfg, const float* w_router, void* w_split,
                              size_t split_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  const size_t need = router_split_bytes(s);
  if (need == 0)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_router_split: this layer shape never uses the tensor-core router");
  MOE_REQUIRE(w_router && w_split, "moe_router_split: NULL pointer");
  MOE_REQUIRE(aligned16(w_router) && aligned16(w_split),
              "moe_router_split: w_router and w_split must be 16-byte aligned");
  MOE_REQUIRE(split_bytes >= need, "moe_router_split: split_bytes %zu < %zu", split_bytes, need);
  cudaError_t err = launch_router_split(s, w_router, w_split, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_router_split launch");
  return MOE_OK;
}

moe_status_t moe_route_ex(const moe_config_t* cfg, const void* x, const float* w_router,
                          const void* w_router_split, const float* logit_bias,
                          int64_t bias_row_stride, float* logits, int32_t* topk_idx,
                          float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(x && w_router && topk_idx && topk_w, "moe_route: NULL input/output pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(w_router), "moe_route: x and w_router must be 16-byte aligned");
  MOE_REQUIRE(w_router_split == nullptr || aligned16(w_router_split),
              "moe_route_ex: w_router_split must be 16-byte aligned");
  MOE_REQUIRE(bias_row_stride == 0 || bias_row_stride >= s.E,
              "moe_route: bias_row_stride must be 0 or >= E");
  float* z = logits;
  if (z == nullptr) z = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + lay.logits);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  if (router_uses_tensor_cores(s)) {
    const char* why = "";
    cudaError_t err = launch_router_tc(
        s, x, w_router, w_router_split, logit_bias, bias_row_stride, logits, z, topk_idx, topk_w,
        static_cast<uint8_t*>(ws) + lay.router_tc,
        reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + lay.partials), ws_status(ws, lay),
        g_wait_ns.load(), strm, &why);
    if (err != cudaSuccess) {
      if (why[0]) return fail(MOE_ERR_CUDA, "moe_route: %s", why);
      return cuda_fail(err, "moe_route (tensor cores) launch");
    }
    return MOE_OK;
  }
  float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + lay.partials);
  cudaError_t err = launch_router(s, x, w_router, logit_bias, bias_row_stride, z, topk_idx, topk_w,
                                  partials, strm);
  if (err != cudaSuccess) return cuda_fail(err, "moe_route launch");
  return MOE_OK;
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                          int32_t* routed_counts, int32_t* kept_counts,
                          int32_t* expert_offsets, int32_t* assign_row,
                          int32_t* token_of_row, void* x_perm, void* ws, size_t ws_bytes,
                          void* stream) {
  MOE_REQUIRE(cfg == nullptr || cfg->drop_policy != MOE_DROP_SCORE,
              "moe_dispatch: MOE_DROP_SCORE needs the selection scores (moe_dispatch_scored)");
  return moe_dispatch_scored(cfg, x, topk_idx, nullptr, nullptr, 0, routed_counts,
                             kept_counts, expert_offsets, assign_row, token_of_row, x_perm, ws,
                             ws_bytes, stream);
}

moe_status_t moe_dispatch_scored(const moe_config_t* cfg, const void* x,
                                 const int32_t* topk_idx, const float* logits,
                                 const float* logit_bias, int64_t bias_row_stride,
                                 int32_t* routed_counts, int32_t* kept_counts,
                                 int32_t* expert_offsets, int32_t* assign_row,
                                 int32_t* token_of_row, void* x_perm, void* ws,
                                 size_t ws_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(topk_idx && routed_counts && kept_counts && expert_offsets && assign_row &&
                  token_of_row && (x || !x_perm),
              "moe_dispatch: NULL pointer");
  MOE_REQUIRE(x_perm == nullptr || (aligned16(x) && aligned16(x_perm)),
              "moe_dispatch: x and x_perm must be 16-byte aligned");
  DispatchScores scores{};
  if (s.drop_policy == MOE_DROP_SCORE) {
    MOE_REQUIRE(logits != nullptr, "moe_dispatch_scored: logits is NULL");
    MOE_REQUIRE(bias_row_stride == 0 || bias_row_stride >= s.E,
                "moe_dispatch_scored: bias_row_stride must be 0 or >= E");
    scores.logits = logits;
    scores.bias = s.bias_mode == MOE_BIAS_SELECTION_ONLY ? logit_bias : nullptr;
    scores.bias_stride = bias_row_stride;
    scores.scratch = static_cast<uint8_t*>(ws) + lay.score;
  }
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + lay.hist);
  cudaError_t err = launch_dispatch(s, x, topk_idx, routed_counts, kept_counts, expert_offsets,
                                    assign_row, token_of_row, x_perm, hist, ws_status(ws, lay),
                                    g_wait_ns.load(), static_cast<cudaStream_t>(stream),
                                    s.drop_policy == MOE_DROP_SCORE ? &scores : nullptr);
  if (err != cudaSuccess) return cuda_fail(err, "moe_dispatch launch");
  return MOE_OK;
}

moe_status_t moe_dispatch_static_scratch(const moe_config_t* cfg, const void* x,
                                         const int32_t* topk_idx, int32_t* routed_counts,
                                         int32_t* kept_counts, int32_t* expert_offsets,
                                         int32_t* assign_row, int32_t* token_of_row,
                                         void* x_perm, void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(x && topk_idx && routed_counts && kept_counts && expert_offsets && assign_row &&
                  token_of_row && x_perm,
              "moe_dispatch_static_scratch: NULL pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(x_perm),
              "moe_dispatch_static_scratch: x and x_perm must be 16-byte aligned");
  if (s.drop_policy == MOE_DROP_SCORE)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_dispatch_static_scratch: MOE_DROP_SCORE needs the selection scores and "
                "workspace scratch (use moe_dispatch_scored)");
  const size_t need = dispatch_hist_bytes(s);
  if (need > kStaticDispatchHistBytes)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_dispatch_static_scratch: ceil(T/%d)*E*4 bytes (times k for pick-rank drops) "
                "= %zu bytes of scratch needed, the fixed scratch holds %zu (use moe_dispatch "
                "with a workspace)",
                kDispatchBlockTokens, need, kStaticDispatchHistBytes);
  cudaError_t err = dispatch_static_scratch(s, x, topk_idx, routed_counts, kept_counts,
                                            expert_offsets, assign_row, token_of_row, x_perm,
                                            g_wait_ns.load(), static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_dispatch_static_scratch");
  return MOE_OK;
}

}  // extern "C"

namespace {

// Both FFN entry points: A rows from x_perm (a_rows == nullptr) or gathered from x.
moe_status_t expert_ffn(const char* name, const moe_config_t* cfg, const void* a,
                        const int32_t* a_rows, const int32_t* expert_offsets,
                        const int32_t* kept_counts, const void* w_gate, const void* w_up,
                        const void* w_down, void* h, void* y_perm, void* ws, size_t ws_bytes,
                        void* stream, const int32_t* comb_token_of_row = nullptr,
                        const int32_t* comb_assign_row = nullptr,
                        const float* comb_topk_w = nullptr, void* comb_out = nullptr) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(a && expert_offsets && kept_counts && w_gate && w_up && w_down && h && y_perm,
              "%s: NULL pointer", name);
  MOE_REQUIRE(aligned16(a) && aligned16(w_gate) && aligned16(w_up) && aligned16(w_down) &&
                  aligned16(h) && aligned16(y_perm),
              "%s: tensors must be 16-byte aligned", name);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t err;
  const bool fuse = comb_out != nullptr;
  if (s.dtype == MOE_F32) {
    err = launch_ffn_simt(s, static_cast<const float*>(a), a_rows, expert_offsets, kept_counts,
                          static_cast<const float*>(w_gate), static_cast<const float*>(w_up),
                          static_cast<const float*>(w_down), static_cast<float*>(h),
                          static_cast<float*>(y_perm), strm);
    if (err != cudaSuccess) return cuda_fail(err, "expert FFN (fp32) launch");
    if (fuse) {  // fp32 layers run the combine kernel after the FFN (same result)
      err = launch_combine(s, y_perm, comb_assign_row, comb_topk_w, comb_out, strm);
      if (err != cudaSuccess) return cuda_fail(err, "combine launch");
    }
    return MOE_OK;
  }
  if (s.d % 64 != 0 || s.f % 64 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "bf16 expert FFN needs d_model and d_ff multiples of 64");
  const char* why = "";
  FusedCombine fc;
  if (fuse) {
    fc.token_of_row = comb_token_of_row;
    fc.assign_row = comb_assign_row;
    fc.topk_w = comb_topk_w;
    fc.arrive = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + lay.arrive);
    fc.out = comb_out;
  }
  err = launch_ffn_tc(s, a, a_rows, expert_offsets, kept_counts, w_gate, w_up, w_down, h, y_perm,
                      ws_status(ws, lay), g_wait_ns.load(), strm, &why, fuse ? &fc : nullptr);
  if (err != cudaSuccess) {
    if (why[0]) return fail(MOE_ERR_CUDA, "%s: %s", name, why);
    return cuda_fail(err, "expert FFN (bf16) launch");
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                            const int32_t* expert_offsets, const int32_t* kept_counts,
                            const void* w_gate, const void* w_up, const void* w_down, void* h,
                            void* y_perm, void* ws, size_t ws_bytes, void* stream) {
  return expert_ffn("moe_expert_ffn", cfg, x_perm, nullptr, expert_offsets, kept_counts, w_gate,
                    w_up, w_down, h, y_perm, ws, ws_bytes, stream);
}

moe_status_t moe_expert_ffn_combine(const moe_config_t* cfg, const void* x, const void* x_perm,
                                    const int32_t* token_of_row, const int32_t* expert_offsets,
                                    const int32_t* kept_counts, const void* w_gate,
                                    const void* w_up, const void* w_down, void* h,
                                    void* y_perm, const int32_t* assign_row,
                                    const float* topk_w, void* out, void* ws, size_t ws_bytes,
                                    void* stream) {
  MOE_REQUIRE(token_of_row && assign_row && topk_w && out && (x || x_perm),
              "moe_expert_ffn_combine: NULL pointer");
  MOE_REQUIRE(aligned16(out), "moe_expert_ffn_combine: out must be 16-byte aligned");
  const void* a = x_perm != nullptr ? x_perm : x;
  const int32_t* a_rows = x_perm != nullptr ? nullptr : token_of_row;
  return expert_ffn("moe_expert_ffn_combine", cfg, a, a_rows, expert_offsets, kept_counts,
                    w_gate, w_up, w_down, h, y_perm, ws, ws_bytes, stream, token_of_row,
                    assign_row, topk_w, out);
}

moe_status_t moe_expert_ffn_gather(const moe_config_t* cfg, const void* x,
                                   const int32_t* token_of_row, const int32_t* expert_offsets,
                                   const int32_t* kept_counts, const void* w_gate,
                                   const void* w_up, const void* w_down, void* h, void* y_perm,
                                   void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(token_of_row != nullptr, "moe_expert_ffn_gather: NULL token_of_row");
  return expert_ffn("moe_expert_ffn_gather", cfg, x, token_of_row, expert_offsets, kept_counts,
                    w_gate, w_up, w_down, h, y_perm, ws, ws_bytes, stream);
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* y_perm,
                         const int32_t* assign_row, const float* topk_w, void* out,
                         void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(y_perm && assign_row && topk_w && out, "moe_combine: NULL pointer");
  MOE_REQUIRE(aligned16(y_perm) && aligned16(out), "moe_combine: y_perm and out must be 16-byte aligned");
  cudaError_t err = launch_combine(s, y_perm, assign_row, topk_w, out,
                                   static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_combine launch");
  return MOE_OK;
}

moe_status_t moe_load_stats(const moe_config_t* cfg, const int32_t* routed_counts,
                            const int32_t* kept_counts, const int32_t* assign_row,
                            moe_load_stats_t* dev_out, moe_load_stats_t* host_out,
                            void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(routed_counts && kept_counts && assign_row && dev_out, "moe_load_stats: NULL pointer");
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t err = launch_stats(s, routed_counts, kept_counts, assign_row, dev_out, strm);
  if (err != cudaSuccess) return cuda_fail(err, "moe_load_stats launch");
  if (host_out != nullptr) {
    err = cudaMemcpyAsync(host_out, dev_out, sizeof(moe_load_stats_t), cudaMemcpyDeviceToHost,
                          strm);
    if (err == cudaSuccess) err = cudaStreamSynchronize(strm);
    if (err != cudaSuccess) return cuda_fail(err, "moe_load_stats copy");
  }
  return MOE_OK;
}

moe_status_t moe_load_stats_merge(const moe_config_t* cfg, const int32_t* routed_sum,
                                  const int32_t* kept_sum, const moe_load_stats_t* parts,
                                  int32_t n_parts, moe_load_stats_t* dev_out,
                                  moe_load_stats_t* host_out, void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(routed_sum && kept_sum && parts && dev_out, "moe_load_stats_merge: NULL pointer");
  MOE_REQUIRE(n_parts >= 1, "moe_load_stats_merge: n_parts must be >= 1");
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t err = launch_stats_merge(s, routed_sum, kept_sum, parts, n_parts, dev_out, strm);
  if (err != cudaSuccess) return cuda_fail(err, "moe_load_stats_merge launch");
  if (host_out != nullptr) {
    err = cudaMemcpyAsync(host_out, dev_out, sizeof(moe_load_stats_t), cudaMemcpyDeviceToHost,
                          strm);
    if (err == cudaSuccess) err = cudaStreamSynchronize(strm);
    if (err != cudaSuccess) return cuda_fail(err, "moe_load_stats_merge copy");
  }
  return MOE_OK;
}

moe_status_t moe_pick_rank_counts(const moe_config_t* cfg, const int32_t* topk_idx,
                                  const int32_t* assign_row, const int32_t* group_of_expert,
                                  int32_t* routed_by_rank, int32_t* kept_by_rank,
                                  int32_t* differs_by_rank, void* ws, size_t ws_bytes,
                                  void* stream) {
  Shape s;
  moe_status_t st = check_config(cfg, &s);
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(topk_idx && assign_row && routed_by_rank && kept_by_rank && differs_by_rank,
              "moe_pick_rank_counts: NULL pointer");
  cudaError_t err = launch_pick_rank_counts(s, topk_idx, assign_row, group_of_expert,
                                            routed_by_rank, kept_by_rank, differs_by_rank,
                                            ws_status(ws, lay), static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_pick_rank_counts launch");
  return MOE_OK;
}

moe_status_t moe_layer_forward(const moe_config_t* cfg, const moe_layer_inputs_t* in,
                               const moe_layer_buffers_t* b, void* ws, size_t ws_bytes,
                               void* stream) {
  MOE_REQUIRE(in != nullptr && b != nullptr, "moe_layer_forward: NULL inputs or buffers");
  moe_status_t st = moe_route_ex(cfg, in->x, in->w_router, in->w_router_split, in->logit_bias,
                                 in->bias_row_stride, b->logits, b->topk_idx, b->topk_w, ws,
                                 ws_bytes, stream);
  if (st != MOE_OK) return st;
  // the logits the router wrote: the caller's array, else the workspace's
  const float* z = b->logits;
  if (z == nullptr) {
    Shape s;
    if ((st = check_config(cfg, &s)) != MOE_OK) return st;
    z = reinterpret_cast<const float*>(static_cast<const uint8_t*>(ws) +
                                       workspace_layout(s).logits);
  }
  st = moe_dispatch_scored(cfg, in->x, b->topk_idx, z, in->logit_bias, in->bias_row_stride,
                           b->routed_counts, b->kept_counts, b->expert_offsets, b->assign_row,
                           b->token_of_row, b->x_perm, ws, ws_bytes, stream);
  if (st != MOE_OK) return st;
  if (b->x_perm != nullptr)
    st = moe_expert_ffn(cfg, b->x_perm, b->expert_offsets, b->kept_counts, in->w_gate,
                        in->w_up, in->w_down, b->h, b->y_perm, ws, ws_bytes, stream);
  else
    st = moe_expert_ffn_gather(cfg, in->x, b->token_of_row, b->expert_offsets, b->kept_counts,
                               in->w_gate, in->w_up, in->w_down, b->h, b->y_perm, ws, ws_bytes,
                               stream);
  if (st != MOE_OK) return st;
  st = moe_combine(cfg, b->y_perm, b->assign_row, b->topk_w, b->out, stream);
  if (st != MOE_OK) return st;
  if (b->stats != nullptr)
    st = moe_load_stats(cfg, b->routed_counts, b->kept_counts, b->assign_row, b->stats, nullptr,
                        stream);
  return st;
}

}  // extern "C"

namespace {

// The EP fields that sizes depend on (everything but the placement pointer).
moe_status_t check_ep_shape(const moe_config_t* cfg, const moe_ep_config_t* ep, Shape* s,
                            const char* name) {
  moe_status_t st = check_config(cfg, s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(ep != nullptr, "%s: ep is NULL", name);
  MOE_REQUIRE(ep->world >= 1 && ep->world <= kMaxDevices, "%s: world must be 1..%d", name,
              kMaxDevices);
  MOE_REQUIRE(ep->rank >= 0 && ep->rank < ep->world, "%s: rank outside [0, world)", name);
  MOE_REQUIRE(ep->ranks_per_node >= 1, "%s: ranks_per_node must be >= 1", name);
  MOE_REQUIRE(ep->n_local >= 1 && ep->n_local <= s->E, "%s: n_local must be 1..E", name);
  MOE_REQUIRE(ep->recv_rows >= 0 && ep->recv_rows <= INT32_MAX,
              "%s: recv_rows must be in [0, 2^31)", name);
  return MOE_OK;
}

moe_status_t check_ep(const moe_config_t* cfg, const moe_ep_config_t* ep, Shape* s,
                      const char* name) {
  moe_status_t st = check_ep_shape(cfg, ep, s, name);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(ep->expert_rank != nullptr, "%s: expert_rank is NULL", name);
  return MOE_OK;
}

int64_t ep_bound(const Shape& s, const moe_ep_config_t* ep) {
  const int64_t per_token = s.k < ep->n_local ? s.k : ep->n_local;
  int64_t per_src = s.T * per_token;
  if (s.C >= 0 && static_cast<int64_t>(ep->n_local) * s.C < per_src)
    per_src = static_cast<int64_t>(ep->n_local) * s.C;
  return per_src * ep->world;
}

}  // namespace

namespace {
// A kernel-recorded status as the call's status and message.
moe_status_t device_error_status(const DevStatus& h) {
  if (h.code == DEV_TIMEOUT)
    return fail(MOE_ERR_TIMEOUT, "a device wait ran out (site %u, item %llu)", h.where,
                (unsigned long long)h.info);
  if (h.code == DEV_RECV_OVERFLOW)
    return fail(MOE_ERR_DEVICE_DATA,
                "expert-parallel row past the receive buffer's recv_rows (pick %llu)",
                (unsigned long long)h.info);
  return fail(MOE_ERR_DEVICE_DATA, "invalid expert index in topk_idx (flat index %llu)",
              (unsigned long long)h.info);
}
}  // namespace

extern "C" {

int64_t moe_ep_recv_rows_bound(const moe_config_t* cfg, const moe_ep_config_t* ep) {
  Shape s;
  if (check_ep_shape(cfg, ep, &s, "moe_ep_recv_rows_bound") != MOE_OK) return -2;
  return ep_bound(s, ep);
}

moe_status_t moe_ep_put_counts(const moe_config_t* cfg, const moe_ep_config_t* ep,
                               const int32_t* kept_counts, int32_t* const* mats, void* stream) {
  Shape s;
  moe_status_t st = check_ep(cfg, ep, &s, "moe_ep_put_counts");
  if (st != MOE_OK) return st;
  MOE_REQUIRE(kept_counts && mats, "moe_ep_put_counts: NULL pointer");
  cudaError_t err = launch_ep_put_counts(s, kept_counts, ep->rank, ep->world, mats,
                                         static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_ep_put_counts launch");
  return MOE_OK;
}

moe_status_t moe_ep_plan(const moe_config_t* cfg, const moe_ep_config_t* ep,
                         const int32_t* count_mat, const int32_t* topk_idx,
                         const int32_t* assign_row, const int32_t* expert_offsets,
                         int32_t* send_row, int32_t* recv_offsets, int32_t* recv_counts,
                         void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_ep(cfg, ep, &s, "moe_ep_plan");
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(count_mat && topk_idx && assign_row && expert_offsets && send_row && recv_offsets &&
                  recv_counts,
              "moe_ep_plan: NULL pointer");
  int32_t* base = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + lay.ep_base);
  cudaError_t err = launch_ep_plan(s, count_mat, ep->expert_rank, ep->world, ep->rank,
                                   ep->n_local, ep->recv_rows, topk_idx, assign_row, expert_offsets, base,
                                   send_row, recv_offsets, recv_counts, ws_status(ws, lay),
                                   static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_ep_plan launch");
  return MOE_OK;
}

moe_status_t moe_ep_dispatch(const moe_config_t* cfg, const moe_ep_config_t* ep,
                             const void* x, const int32_t* topk_idx, const int32_t* send_row,
                             void* const* recv, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_ep(cfg, ep, &s, "moe_ep_dispatch");
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(x && topk_idx && send_row && recv, "moe_ep_dispatch: NULL pointer");
  MOE_REQUIRE(aligned16(x), "moe_ep_dispatch: x must be 16-byte aligned");
  cudaError_t err = launch_ep_dispatch(s, x, topk_idx, send_row, ep->expert_rank, ep->world,
                                       recv, ep->recv_rows, ws_status(ws, lay),
                                       static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_ep_dispatch launch");
  return MOE_OK;
}

moe_status_t moe_ep_expert_ffn(const moe_config_t* cfg, const moe_ep_config_t* ep,
                               const void* recv_x, const int32_t* recv_offsets,
                               const int32_t* recv_counts, const void* w_gate_local,
                               const void* w_up_local, const void* w_down_local, void* h,
                               void* y_recv, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_ep(cfg, ep, &s, "moe_ep_expert_ffn");
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(recv_x && recv_offsets && recv_counts && w_gate_local && w_up_local &&
                  w_down_local && h && y_recv,
              "moe_ep_expert_ffn: NULL pointer");
  MOE_REQUIRE(aligned16(recv_x) && aligned16(w_gate_local) && aligned16(w_up_local) &&
                  aligned16(w_down_local) && aligned16(h) && aligned16(y_recv),
              "moe_ep_expert_ffn: tensors must be 16-byte aligned");
  if (ep->recv_rows == 0) return MOE_OK;
  // the local grouped GEMM: n_local buckets in a buffer of recv_rows rows; a bucket holds
  // at most world x min(T, C) rows
  Shape sl = s;
  sl.E = ep->n_local;
  sl.max_rows = ep->recv_rows;
  sl.T = s.T * ep->world;
  sl.C = s.C >= 0 ? s.C * ep->world : -1;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (s.dtype == MOE_F32) {
    err = launch_ffn_simt(sl, static_cast<const float*>(recv_x), nullptr, recv_offsets,
                          recv_counts, static_cast<const float*>(w_gate_local),
                          static_cast<const float*>(w_up_local),
                          static_cast<const float*>(w_down_local), static_cast<float*>(h),
                          static_cast<float*>(y_recv), strm);
    if (err != cudaSuccess) return cuda_fail(err, "moe_ep_expert_ffn (fp32) launch");
    return MOE_OK;
  }
  if (s.d % 64 != 0 || s.f % 64 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "bf16 expert FFN needs d_model and d_ff multiples of 64");
  const char* why = "";
  err = launch_ffn_tc(sl, recv_x, nullptr, recv_offsets, recv_counts, w_gate_local, w_up_local,
                      w_down_local, h, y_recv, ws_status(ws, lay), g_wait_ns.load(), strm, &why);
  if (err != cudaSuccess) {
    if (why[0]) return fail(MOE_ERR_CUDA, "moe_ep_expert_ffn: %s", why);
    return cuda_fail(err, "moe_ep_expert_ffn (bf16) launch");
  }
  return MOE_OK;
}

moe_status_t moe_ep_combine(const moe_config_t* cfg, const moe_ep_config_t* ep,
                            const void* const* ybuf, const int32_t* topk_idx,
                            const int32_t* send_row, const float* topk_w, void* out,
                            void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  moe_status_t st = check_ep(cfg, ep, &s, "moe_ep_combine");
  if (st != MOE_OK) return st;
  WsLayout lay;
  if ((st = check_ws(s, ws, ws_bytes, &lay)) != MOE_OK) return st;
  MOE_REQUIRE(ybuf && topk_idx && send_row && topk_w && out, "moe_ep_combine: NULL pointer");
  MOE_REQUIRE(aligned16(out), "moe_ep_combine: out must be 16-byte aligned");
  cudaError_t err = launch_ep_combine(s, ybuf, topk_idx, send_row, ep->expert_rank, ep->world,
                                      ep->recv_rows, topk_w, out,
                                      static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_ep_combine launch");
  return MOE_OK;
}

moe_status_t moe_ep_stats(const moe_config_t* cfg, const moe_ep_config_t* ep,
                          const int32_t* count_mat, moe_ep_stats_t* dev_out,
                          moe_ep_stats_t* host_out, void* stream) {
  Shape s;
  moe_status_t st = check_ep(cfg, ep, &s, "moe_ep_stats");
  if (st != MOE_OK) return st;
  MOE_REQUIRE(count_mat && dev_out, "moe_ep_stats: NULL pointer");
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t err = launch_ep_stats(s, count_mat, ep->expert_rank, ep->world,
                                    ep->ranks_per_node, dev_out, strm);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ep_stats launch");
  if (host_out != nullptr) {
    err = cudaMemcpyAsync(host_out, dev_out, sizeof(moe_ep_stats_t), cudaMemcpyDeviceToHost,
                          strm);
    if (err == cudaSuccess) err = cudaStreamSynchronize(strm);
    if (err != cudaSuccess) return cuda_fail(err, "moe_ep_stats host copy");
  }
  return MOE_OK;
}

moe_status_t moe_ipc_handle(const void* dev_ptr, unsigned char handle_out[64],
                            int64_t* offset_out) {
  MOE_REQUIRE(dev_ptr && handle_out && offset_out, "moe_ipc_handle: NULL pointer");
  typedef CUresult (*RangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
  static RangeFn range = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      range = reinterpret_cast<RangeFn>(fn);
  });
  if (range == nullptr)
    return fail(MOE_ERR_CUDA, "moe_ipc_handle: cuMemGetAddressRange is not available");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return fail(MOE_ERR_CUDA, "moe_ipc_handle: pointer is not device memory of this process");
  cudaIpcMemHandle_t hnd;
  cudaError_t err = cudaIpcGetMemHandle(&hnd, reinterpret_cast<void*>(base));
  if (err != cudaSuccess) return cuda_fail(err, "moe_ipc_handle");
  static_assert(sizeof(hnd) == 64, "CUDA IPC handles are 64 bytes");
  memcpy(handle_out, &hnd, sizeof(hnd));
  *offset_out = static_cast<int64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return MOE_OK;
}

moe_status_t moe_ipc_open(const unsigned char handle[64], void** dev_ptr_out) {
  MOE_REQUIRE(handle && dev_ptr_out, "moe_ipc_open: NULL pointer");
  cudaIpcMemHandle_t hnd;
  memcpy(&hnd, handle, sizeof(hnd));
  cudaError_t err = cudaIpcOpenMemHandle(dev_ptr_out, hnd, cudaIpcMemLazyEnablePeerAccess);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ipc_open");
  return MOE_OK;
}

moe_status_t moe_ipc_close(void* dev_ptr) {
  MOE_REQUIRE(dev_ptr, "moe_ipc_close: NULL pointer");
  cudaError_t err = cudaIpcCloseMemHandle(dev_ptr);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ipc_close");
  return MOE_OK;
}

moe_status_t moe_check_device_error(void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(ws != nullptr && ws_bytes >= sizeof(DevStatus), "moe_check_device_error: bad workspace");
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaStreamSynchronize(strm);
  if (err != cudaSuccess) return cuda_fail(err, "moe_check_device_error sync");
  DevStatus h;
  err = cudaMemcpy(&h, ws, sizeof(DevStatus), cudaMemcpyDeviceToHost);
  if (err != cudaSuccess) return cuda_fail(err, "moe_check_device_error read");
  if (h.code == DEV_OK) return MOE_OK;
  err = cudaMemset(ws, 0, sizeof(DevStatus));
  if (err != cudaSuccess) return cuda_fail(err, "moe_check_device_error clear");
  return device_error_status(h);
}

moe_status_t moe_static_scratch_check(void* stream) {
  DevStatus h;
  cudaError_t err = static_scratch_status(&h, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_static_scratch_check");
  if (h.code == DEV_OK) return MOE_OK;
  return device_error_status(h);
}

moe_status_t moe_selftest_bounded_wait(void* ws, size_t ws_bytes, void* stream) {
  MOE_REQUIRE(ws != nullptr && ws_bytes >= sizeof(DevStatus), "moe_selftest_bounded_wait: bad workspace");
  cudaError_t err = launch_wait_selftest(static_cast<DevStatus*>(ws), g_wait_ns.load(),
                                         static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_selftest_bounded_wait launch");
  return MOE_OK;
}

}  // extern "C"
