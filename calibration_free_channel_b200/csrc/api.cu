// api.cu -- the C ABI (include/moe_reader.h): argument validation, workspace
// carving and launches.  Every check runs on the host before anything is
// enqueued.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/moe_reader.h"
#include "common.cuh"
#include "kernels.h"

namespace {

thread_local std::string g_err;

moe_status fail(moe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

moe_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

#define REQUIRE(cond, ...) \
  do {                     \
    if (!(cond)) return fail(MOE_EINVAL, __VA_ARGS__); \
  } while (0)
#define REQUIRE_PTR(p)                                                          \
  do {                                                                          \
    if (!(p)) return fail(MOE_EINVAL, "%s is NULL", #p);                        \
    if (!aligned16(p)) return fail(MOE_EINVAL, "%s is not 16-byte aligned", #p); \
  } while (0)
#define OPT_PTR(p)                                                              \
  do {                                                                          \
    if ((p) && !aligned16(p)) return fail(MOE_EINVAL, "%s is not 16-byte aligned", #p); \
  } while (0)

// The device address of page-locked host memory the current device can
// address directly, or nullptr (pageable memory, or a query failure).
void* device_view(const void* host) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

moe_status check_shape(int B, int E, int top_e, int I, int d) {
  REQUIRE(B >= 1 && B <= 256, "B = %d outside [1, 256]", B);
  REQUIRE(E >= 1 && E <= 1024, "E = %d outside [1, 1024]", E);
  REQUIRE(top_e >= 1 && top_e <= 16 && top_e <= E, "top_e = %d outside [1, min(E, 16)]", top_e);
  REQUIRE(I >= 16 && I <= 2048, "I = %d outside [16, 2048]", I);
  REQUIRE(pow2(d) && d >= 256 && d <= 4096, "d = %d is not a power of two in [256, 4096]", d);
  return MOE_OK;
}

moe_status check_layer(const moe_reader_layer* L, bool sparse) {
  REQUIRE(L != nullptr, "layer is NULL");
  REQUIRE(L->cluster_size == 0 || (L->cluster_size >= 2 && L->cluster_size <= 16),
          "cluster_size = %d: use 0 (automatic) or 2 .. 16", L->cluster_size);
  REQUIRE_PTR(L->w_router);
  OPT_PTR(L->router_bias);
  REQUIRE_PTR(L->w_gate);
  REQUIRE_PTR(L->w_up);
  REQUIRE_PTR(L->w_down);
  OPT_PTR(L->expert_slot);
  if (sparse) {
    REQUIRE_PTR(L->rot_sign);
    REQUIRE_PTR(L->sk_gate);
    REQUIRE_PTR(L->sk_up);
    REQUIRE(L->sketch_format == 0 || L->sketch_format == 1,
            "sketch_format = %d: use 0 (2-bit codes) or 1 (base 3, five trits per byte)", L->sketch_format);
    REQUIRE_PTR(L->alpha_gate);
    REQUIRE_PTR(L->alpha_up);
    REQUIRE(L->recovery_input == 0 || L->recovery_input == 1, "recovery_input = %d: use 0 or 1", L->recovery_input);
    REQUIRE(L->path >= 0 && L->path <= 2, "path = %d: use 0 (automatic), 1 (one cluster per expert) or 2 (streamed)",
            L->path);
    REQUIRE(L->r >= 0 && L->r <= 128 && L->r % 8 == 0 && L->r <= L->I, "r = %d: need r in {0, 8, ..., 128}, r <= I",
            L->r);
    if (L->r > 0) {
      REQUIRE_PTR(L->u_sigma);
      REQUIRE_PTR(L->v);
    }
  }
  return MOE_OK;
}

// ep_size > 0: expert-parallel step of rank ep_rank; writes y_partial (fp32)
// instead of y.  clear_counters: after validation, before any launch, zero
// the workspace's combine counters (the noalloc entry's shared scratch).
// A copy enqueued after validation and before the step's first launch (the
// host-buffer entry's input).
struct PreCopy {
  const void* src;
  void* dst;
  size_t bytes;
  bool kernel;  // true: a copy kernel (src device-accessible); false: cudaMemcpyAsync
};

moe_status run_forward(const moe_reader_layer* L, int B, int k, int c, const uint16_t* x, const uint16_t* residual,
                       uint16_t* y, const moe_reader_debug* dbg, void* workspace, size_t ws_bytes, void* stream,
                       bool dense, int ep_rank = 0, int ep_size = 0, float* y_partial = nullptr,
                       bool clear_counters = false, const PreCopy* pre = nullptr) {
  moe_status st = check_layer(L, !dense);
  if (st != MOE_OK) return st;
  st = check_shape(B, L->E, L->top_e, L->I, L->d);
  if (st != MOE_OK) return st;
  if (!dense) {
    REQUIRE(k >= 1 && k <= L->I, "k = %d outside [1, I = %d]", k, L->I);
    REQUIRE(c >= k && c <= L->I, "c = %d outside [k = %d, I = %d]", c, k, L->I);
  }
  REQUIRE_PTR(x);
  if (dbg) REQUIRE(dbg->withhold_copy == 0 || dbg->withhold_copy == 1, "withhold_copy = %d: use 0 or 1",
                   dbg->withhold_copy);
  if (ep_size > 0) {
    REQUIRE(ep_size <= L->E && ep_rank >= 0 && ep_rank < ep_size, "ep_rank = %d, ep_size = %d: need 0 <= rank < size <= E",
            ep_rank, ep_size);
    REQUIRE_PTR(y_partial);
  } else {
    REQUIRE_PTR(y);
  }
  OPT_PTR(residual);
  REQUIRE_PTR(workspace);
  const int sI = dense ? 0 : L->I, sr = dense ? 0 : L->r;
  const size_t need = moe::workspace_layout(B, L->E, L->top_e, L->d, sI, sr, nullptr, nullptr);
  REQUIRE(ws_bytes >= need, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  if (L->expert_slot && (dense || L->path == 1))
    return fail(MOE_EUNSUPPORTED, "expert_slot (held experts only) is read by the streamed reader (path 0 or 2)");
  const bool streamed = !dense && (ep_size > 0 || L->path == 2 || L->expert_slot ||
                                   (L->path == 0 && !moe::reader_supports(B, L->d)));
  if (!dense && !streamed && !moe::reader_supports(B, L->d))
    return fail(MOE_EUNSUPPORTED, "path 1 (one cluster per expert) runs B <= 2 and d <= 2048 (B = %d, d = %d)", B,
                L->d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe::Workspace ws;
  moe::workspace_layout(B, L->E, L->top_e, L->d, sI, sr, workspace, &ws);
  if (clear_counters) {
    const cudaError_t ce = cudaMemsetAsync(ws.counters, 0, sizeof(unsigned) * moe::kMaxTokens * moe::kMaxCluster, s);
    if (ce != cudaSuccess) return cuda_fail(ce, "clearing the combine counters");
  }
  if (pre) {
    const cudaError_t ce = pre->kernel ? moe::launch_copy16(pre->src, pre->dst, pre->bytes, s)
                                       : cudaMemcpyAsync(pre->dst, pre->src, pre->bytes, cudaMemcpyHostToDevice, s);
    if (ce != cudaSuccess) return cuda_fail(ce, "host-to-device copy");
  }

  moe::RouteArgs ra = {};
  ra.B = B;
  ra.E = L->E;
  ra.d = L->d;
  ra.top_e = L->top_e;
  ra.x = x;
  ra.w_router = L->w_router;
  ra.bias = L->router_bias;
  ra.rot_sign = L->rot_sign;
  ra.ws = ws;
  ra.dbg_ids = dbg ? dbg->ids : nullptr;
  ra.dbg_w = dbg ? dbg->weights : nullptr;
  ra.quantize = !dense;
  cudaError_t e = cudaSuccess;
  ra.ep_rank = ep_rank;
  ra.ep_size = ep_size;
  ra.expert_slot = L->expert_slot;
  // steps of at most two tokens route inside the cluster kernels
  if (!moe::fused_routing(B) || streamed) {
    e = moe::launch_route(ra, s);
    if (e != cudaSuccess) return cuda_fail(e, "route launch");
  }

  moe::ExpertArgs a = {};
  a.B = B;
  a.E = L->E;
  a.top_e = L->top_e;
  a.I = L->I;
  a.d = L->d;
  a.k = k;
  a.c = c;
  a.r = dense ? 0 : L->r;
  a.recovery_input = dense ? 0 : L->recovery_input;
  a.ep_partial = ep_size > 0 ? 1 : 0;
  a.cs = 0;  // chosen at launch
  a.force_cs = L->cluster_size;
  a.wait_ns = dbg && dbg->wait_limit_us ? 1000ull * dbg->wait_limit_us : moe::kWaitLimitNs;
  a.withhold_copy = dbg ? dbg->withhold_copy : 0;
  a.nmax = B < moe::kMaxGroup ? B : moe::kMaxGroup;
  a.x = x;
  a.w_router = L->w_router;
  a.bias = L->router_bias;
  a.rot_sign = L->rot_sign;
  a.w_gate = L->w_gate;
  a.w_up = L->w_up;
  a.w_down = L->w_down;
  a.sk_gate = static_cast<const uint32_t*>(L->sk_gate);
  a.sk_up = static_cast<const uint32_t*>(L->sk_up);
  a.sk3 = dense ? 0 : L->sketch_format;
  a.alpha_gate = L->alpha_gate;
  a.alpha_up = L->alpha_up;
  a.u_sigma = L->u_sigma;
  a.v = L->v;
  a.residual = residual;
  a.y = y;
  a.ws = ws;
  if (dbg) {
    a.dbg_ids = dbg->ids;
    a.dbg_w = dbg->weights;
    a.dbg_G = dbg->dot_gate;
    a.dbg_U = dbg->dot_up;
    a.dbg_sigma = dbg->score;
    a.dbg_cand = dbg->cand;
    a.dbg_kept = dbg->kept;
    a.dbg_a_kept = dbg->a_kept;
    a.dbg_y_expert = dbg->y_expert;
    a.dbg_phase = reinterpret_cast<unsigned long long*>(dbg->phase_ns);
  }
  cudaEvent_t ev_before = dbg ? static_cast<cudaEvent_t>(dbg->ev_before) : nullptr;
  cudaEvent_t ev_after = dbg ? static_cast<cudaEvent_t>(dbg->ev_after) : nullptr;
  if (ev_before) cudaEventRecord(ev_before, s);
  e = dense ? moe::launch_dense(a, s) : streamed ? moe::launch_stream(a, s) : moe::launch_reader(a, s);
  if (e != cudaSuccess) return cuda_fail(e, dense ? "dense expert launch" : "reader launch");
  if (ep_size > 0) {
    e = moe::launch_ep_combine(B, L->top_e, L->d, ep_rank, ep_size, ws, y_partial, s);
    if (e != cudaSuccess) return cuda_fail(e, "expert-parallel combine launch");
  }
  if (ev_after) cudaEventRecord(ev_after, s);
  return MOE_OK;
}

}  // namespace

moe_status moe::set_last_error(moe_status st, const char* msg) {
  g_err = msg;
  return st;
}

moe_status moe::forward_scratch(const moe_reader_layer* layer, int B, int k, int c, const uint16_t* x,
                                const uint16_t* residual, uint16_t* y, void* scratch, size_t bytes, void* stream) {
  return run_forward(layer, B, k, c, x, residual, y, nullptr, scratch, bytes, stream, false, 0, 0, nullptr, true);
}

extern "C" {

size_t moe_reader_workspace_bytes(int B, int E, int top_e, int I, int d, int k, int c, int r) {
  (void)k;
  (void)c;
  if (B < 1 || E < 1 || top_e < 1 || d < 1 || I < 0 || r < 0) return 0;
  return moe::workspace_layout(B, E, top_e, d, I, r, nullptr, nullptr);
}

moe_status moe_reader_build_sketch(int E, int I, int d, const uint16_t* w_gate, const uint16_t* w_up,
                                   uint64_t rot_seed, int8_t* rot_sign, uint32_t* sk_gate, uint32_t* sk_up,
                                   float* alpha_gate, float* alpha_up, void* stream) {
  moe_status st = check_shape(1, E, 1, I, d);
  if (st != MOE_OK) return st;
  REQUIRE_PTR(w_gate);
  REQUIRE_PTR(w_up);
  REQUIRE_PTR(rot_sign);
  REQUIRE_PTR(sk_gate);
  REQUIRE_PTR(sk_up);
  REQUIRE_PTR(alpha_gate);
  REQUIRE_PTR(alpha_up);
  cudaError_t e = moe::launch_build_sketch(E, I, d, w_gate, w_up, rot_seed, rot_sign, sk_gate, sk_up, alpha_gate,
                                           alpha_up, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "build_sketch launch");
}

size_t moe_reader_sketch_row_bytes(int d, int format) {
  if (d < 16 || d % 16 != 0) return 0;
  if (format == 0) return (size_t)d / 4;
  if (format == 1) return (size_t)moe::sk3_row_bytes(d);
  return 0;
}

moe_status moe_reader_sketch_to_base3(int E, int I, int d, const uint32_t* sk_codes, uint8_t* sk_base3,
                                      void* stream) {
  moe_status st = check_shape(1, E, 1, I, d);
  if (st != MOE_OK) return st;
  REQUIRE_PTR(sk_codes);
  REQUIRE_PTR(sk_base3);
  cudaError_t e = moe::launch_sketch_to_base3((long)E * I, d, sk_codes, sk_base3, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "sketch_to_base3 launch");
}

size_t moe_reader_lowrank_workspace_bytes(int E, int I, int d, int r) {
  if (E < 1 || I < 1 || d < 1 || r < 1) return 0;
  return moe::lowrank_ws_bytes(E, I, d, r);
}

moe_status moe_reader_build_lowrank(int E, int I, int d, int r, const uint16_t* w_down, uint16_t* u_sigma,
                                    uint16_t* v, void* workspace, size_t ws_bytes, void* stream) {
  moe_status st = check_shape(1, E, 1, I, d);
  if (st != MOE_OK) return st;
  REQUIRE(r >= 8 && r <= 128 && r % 8 == 0 && r <= I, "r = %d: need r in {8, ..., 128}, r <= I", r);
  if (r > 64) return fail(MOE_EUNSUPPORTED, "build_lowrank supports r <= 64 (got %d)", r);
  const int p = I < r + 32 ? I : r + 32;
  const size_t sm1 = sizeof(float) * I * 16 + 2 * sizeof(double) * p * p;
  const size_t sm2 = sizeof(float) * (size_t)I * r;
  if (sm1 > 227 * 1024 || sm2 > 227 * 1024)
    return fail(MOE_EUNSUPPORTED, "build_lowrank: I = %d, r = %d exceed this build's shared-memory plan", I, r);
  REQUIRE_PTR(w_down);
  REQUIRE_PTR(u_sigma);
  REQUIRE_PTR(v);
  REQUIRE_PTR(workspace);
  const size_t need = moe::lowrank_ws_bytes(E, I, d, r);
  REQUIRE(ws_bytes >= need, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  cudaError_t e =
      moe::launch_build_lowrank(E, I, d, r, w_down, u_sigma, v, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "build_lowrank launch");
}

moe_status moe_reader_forward(const moe_reader_layer* layer, int B, int k, int c, const uint16_t* x,
                              const uint16_t* residual, uint16_t* y, const moe_reader_debug* dbg, void* workspace,
                              size_t ws_bytes, void* stream) {
  return run_forward(layer, B, k, c, x, residual, y, dbg, workspace, ws_bytes, stream, false);
}

moe_status moe_reader_forward_ep(const moe_reader_layer* layer, int B, int k, int c, const uint16_t* x, int ep_rank,
                                 int ep_size, float* y_partial, const moe_reader_debug* dbg, void* workspace,
                                 size_t ws_bytes, void* stream) {
  REQUIRE(ep_size >= 1, "ep_size = %d must be >= 1", ep_size);
  return run_forward(layer, B, k, c, x, nullptr, nullptr, dbg, workspace, ws_bytes, stream, false, ep_rank, ep_size,
                     y_partial);
}

moe_status moe_reader_ep_finish(int B, int d, const float* y_sum, const uint16_t* residual, uint16_t* y,
                                void* stream) {
  REQUIRE(B >= 1 && B <= 256, "B = %d outside [1, 256]", B);
  REQUIRE(d >= 1 && d <= 4096, "d = %d outside [1, 4096]", d);
  REQUIRE_PTR(y_sum);
  REQUIRE_PTR(y);
  OPT_PTR(residual);
  cudaError_t e = moe::launch_ep_finish(B, d, y_sum, residual, y, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "expert-parallel finish launch");
}

moe_status moe_reader_forward_dense(const moe_reader_layer* layer, int B, const uint16_t* x, const uint16_t* residual,
                                    uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
  return run_forward(layer, B, 1, 1, x, residual, y, nullptr, workspace, ws_bytes, stream, true);
}

moe_status moe_reader_forward_host(const moe_reader_layer* layer, int B, int k, int c, const uint16_t* x_host,
                                   uint16_t* x_dev, uint16_t* y_dev, uint16_t* y_host, void* workspace,
                                   size_t ws_bytes, void* stream) {
  REQUIRE(layer != nullptr, "layer is NULL");
  REQUIRE(x_host != nullptr && y_host != nullptr, "host buffers must not be NULL");
  REQUIRE(B >= 1 && B <= 256, "B = %d outside [1, 256]", B);
  REQUIRE_PTR(x_dev);
  REQUIRE_PTR(y_dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(uint16_t) * (size_t)B * layer->d;
  // Pinned host buffers the device can address (page-locked memory under
  // unified addressing) move through small copy kernels on the SMs: for a few
  // kilobytes that is several microseconds faster than a DMA-engine copy, and
  // the copies chain with the step's kernels by programmatic dependent launch.
  // Other host memory takes cudaMemcpyAsync.
  const void* xsrc = device_view(x_host);
  void* ydst = device_view(y_host);
  const bool fast = xsrc && ydst && bytes % 16 == 0 && aligned16(xsrc) && aligned16(ydst);
  const PreCopy pre = {fast ? xsrc : x_host, x_dev, bytes, fast};
  moe_status st =
      run_forward(layer, B, k, c, x_dev, nullptr, y_dev, nullptr, workspace, ws_bytes, stream, false, 0, 0, nullptr,
                  false, &pre);
  if (st != MOE_OK) return st;
  const cudaError_t e = fast ? moe::launch_copy16(y_dev, ydst, bytes, s)
                             : cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "device-to-host copy");
}

moe_status moe_reader_rmsnorm(int B, int d, float eps, const uint16_t* x, uint16_t* h, void* stream) {
  REQUIRE(B >= 1 && B <= 65535, "B = %d outside [1, 65535]", B);
  REQUIRE(d >= 1 && d % 8 == 0, "d = %d must be a positive multiple of 8", d);
  REQUIRE(eps >= 0.0f, "eps must be >= 0");
  REQUIRE_PTR(x);
  REQUIRE_PTR(h);
  cudaError_t e = moe::launch_rmsnorm(B, d, eps, x, h, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "rmsnorm launch");
}

moe_status moe_reader_check_error(void* workspace, void* stream) {
  if (!workspace) {
    // the noalloc entry's scratch on the current device
    cudaError_t se = cudaSuccess;
    workspace = moe::noalloc_scratch(&se);
    if (!workspace) return cuda_fail(se, "scratch set-up (cudaGetSymbolAddress)");
  }
  REQUIRE_PTR(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  moe::Workspace ws;
  moe::workspace_layout(1, 1, 1, 16, 0, 0, workspace, &ws);  // err sits at offset 0 for every shape
  uint32_t word = 0;
  e = cudaMemcpy(&word, ws.err, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "error word read");
  if (word == 0) return MOE_OK;
  const uint32_t zero = 0;
  cudaMemcpy(ws.err, &zero, sizeof zero, cudaMemcpyHostToDevice);
  return fail((word & moe::kErrCopyTimeout) ? MOE_ETIMEOUT : MOE_EDEVICE,
              "device error word 0x%x (1: a bounded copy wait ran out; 2: bad work item; 4: a routed expert has no "
              "weight slot)",
              word);
}

moe_status moe_reader_launch_plan(int dense, int B, int E, int top_e, int I, int d, int r, int32_t* out4) {
  moe_status st = check_shape(B, E, top_e, I, d);
  if (st != MOE_OK) return st;
  REQUIRE(out4 != nullptr, "out4 is NULL");
  moe::ExpertArgs a = {};
  a.B = B;
  a.E = E;
  a.top_e = top_e;
  a.I = I;
  a.d = d;
  a.r = dense ? 0 : r;
  a.nmax = B < moe::kMaxGroup ? B : moe::kMaxGroup;
  a.ws.max_items = moe::max_work_items(B, E, top_e, moe::kMaxGroup);
  int o[4];
  cudaError_t e = moe::query_plan(a, dense != 0, o);
  if (e != cudaSuccess) return cuda_fail(e, "launch plan");
  for (int i = 0; i < 4; i++) out4[i] = o[i];
  return MOE_OK;
}

const char* moe_reader_last_error(void) { return g_err.c_str(); }

}  // extern "C"
