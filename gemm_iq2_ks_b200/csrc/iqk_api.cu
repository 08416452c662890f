// C ABI of the library (declared and documented in include/iqk.h).
// Host-side argument validation, workspace checks and dispatch; no entry
// point allocates, frees or synchronises except iqk_moe_status, which reads
// the status word back by design.
#include <stdio.h>
#include <string.h>

#include "iqk.h"
#include "iqk_internal.h"

using namespace iqk;

namespace {

thread_local char g_cuda_err[256] = "";

int cuda_fail(cudaError_t e) {
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return IQK_ECUDA;
}

// Launch helpers return -4 on a CUDA failure; record the text.
int from_launch(int rc) {
  if (rc == -4) {
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaErrorUnknown;
    return cuda_fail(e);
  }
  return rc;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  static int cached[64] = {0};
  if (dev < 0 || dev >= 64) return -1;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cached[dev] = n;
  }
  return cached[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_weights(const iqk_weights* w, WDev* out) {
  if (!w) return IQK_EINVAL;
  if (w->fmt != IQK_IQ2_KS && w->fmt != IQK_IQ2_K) return IQK_EINVAL;
  if (w->experts < 1 || w->rows < 1) return IQK_ESHAPE;
  if (w->cols <= 0 || w->cols % 256) return IQK_ESHAPE;
  if (!w->qs || !w->scl || !w->sex || !w->dv) return IQK_EINVAL;
  if ((w->fmt == IQK_IQ2_KS) != (w->sch != nullptr)) return IQK_EINVAL;
  // planes are staged by TMA / bulk copies: every base 16-byte aligned
  if (!aligned(w->qs, 16) || !aligned(w->scl, 16) || !aligned(w->sex, 16) || !aligned(w->dv, 16)) return IQK_EINVAL;
  if (w->sch && !aligned(w->sch, 16)) return IQK_EINVAL;
  if ((int64_t)w->experts * w->rows >= (int64_t)1 << 31) return IQK_ESHAPE;
  if (w->slots && !aligned(w->slots, 16)) return IQK_EINVAL;
  out->qs = w->qs;
  out->scl = w->scl;
  out->sch = w->sch;
  out->sex = w->sex;
  out->dv = w->dv;
  out->slots = w->slots;
  out->experts = w->experts;
  out->rows = w->rows;
  out->cols = w->cols;
  return IQK_OK;
}

int check_values(const float* values, Values* V) {
  if (!values) return IQK_EINVAL;
  memcpy(V->v, values, sizeof(V->v));
  return IQK_OK;
}

int check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return IQK_OK;
  if (!ws || !aligned(ws, 256) || have < need) return IQK_EWORKSPACE;
  return IQK_OK;
}

int check_moe(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down, WDev* g, WDev* u,
              WDev* d) {
  int rc;
  if ((rc = check_weights(gate, g)) || (rc = check_weights(up, u)) || (rc = check_weights(down, d))) return rc;
  if (g->experts != u->experts || g->experts != d->experts) return IQK_EINVAL;
  if (g->rows != u->rows || g->cols != u->cols) return IQK_EINVAL;
  if (d->rows != g->cols || d->cols != g->rows) return IQK_EINVAL;
  if (g->rows % 256) return IQK_ESHAPE;  // inter is the down projection's reduction width
  return IQK_OK;
}

}  // namespace

extern "C" {

const char* iqk_strerror(int s) {
  switch (s) {
    case IQK_OK: return "ok";
    case IQK_EINVAL: return "invalid argument";
    case IQK_ESHAPE: return "unsupported shape (widths must be positive multiples of 256)";
    case IQK_EUNSUPPORTED: return "unsupported configuration";
    case IQK_ECUDA: return "CUDA error";
    case IQK_ETIMEOUT: return "bounded device wait expired";
    case IQK_EWORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
  }
}

const char* iqk_last_cuda_error(void) { return g_cuda_err; }

int iqk_version(void) { return 2; }

int64_t iqk_row_bytes(int32_t fmt, int32_t cols) {
  if (cols <= 0 || cols % 256) return -1;
  if (fmt == IQK_IQ2_KS) return 2 + (int64_t)70 * cols / 256;
  if (fmt == IQK_IQ2_K) return (int64_t)76 * cols / 256;
  return -1;
}

size_t iqk_slots_bytes(const iqk_weights* w) {
  WDev wd;
  if (check_weights(w, &wd)) return 0;
  return slots_bytes(wd, w->fmt);
}

int iqk_pack_slots(const iqk_weights* w, uint8_t* out, size_t out_bytes, void* stream) {
  WDev wd;
  int rc;
  if ((rc = check_weights(w, &wd))) return rc;
  wd.slots = nullptr;  // packed from the planes
  if (!out || !aligned(out, 16) || out_bytes < slots_bytes(wd, w->fmt)) return IQK_EWORKSPACE;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_pack_slots(wd, w->fmt, out, (cudaStream_t)stream, sms));
}

int iqk_prefill_a_tile(const iqk_weights* w, int32_t expert, int32_t row0, int32_t nrows, const float* values,
                       uint16_t* out, void* stream) {
  WDev wd;
  Values V;
  int rc;
  if ((rc = check_weights(w, &wd)) || (rc = check_values(values, &V))) return rc;
  if (expert < 0 || expert >= wd.experts || row0 < 0 || nrows < 1 || (int64_t)row0 + nrows > wd.rows) return IQK_EINVAL;
  if (!out || !aligned(out, 16)) return IQK_EINVAL;
  return from_launch(launch_pf_a_tile(wd, w->fmt, expert, row0, nrows, V, out, (cudaStream_t)stream));
}

int iqk_dequant(const iqk_weights* w, int32_t expert, const float* values, float* out, void* stream) {
  WDev wd;
  Values V;
  int rc;
  if ((rc = check_weights(w, &wd)) || (rc = check_values(values, &V))) return rc;
  if (expert < 0 || expert >= wd.experts || !out || !aligned(out, 16)) return IQK_EINVAL;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_dequant(wd, w->fmt, expert, V, out, false, false, (cudaStream_t)stream, sms));
}

int iqk_dequant_bf16(const iqk_weights* w, int32_t expert, const float* values, uint16_t* out, void* stream) {
  WDev wd;
  Values V;
  int rc;
  if ((rc = check_weights(w, &wd)) || (rc = check_values(values, &V))) return rc;
  if (expert < 0 || expert >= wd.experts || !out || !aligned(out, 16)) return IQK_EINVAL;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_dequant(wd, w->fmt, expert, V, out, true, false, (cudaStream_t)stream, sms));
}

int iqk_dequant_floor(const iqk_weights* w, int32_t expert, int32_t bf16, uint32_t* out, void* stream) {
  WDev wd;
  int rc;
  if ((rc = check_weights(w, &wd))) return rc;
  if (expert < 0 || expert >= wd.experts || !out || !aligned(out, 16)) return IQK_EINVAL;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  Values V{};
  return from_launch(launch_dequant(wd, w->fmt, expert, V, out, bf16 != 0, true, (cudaStream_t)stream, sms));
}

size_t iqk_gemv_workspace_bytes(int32_t T, int32_t rows, int32_t cols) {
  if (T < 1 || T > 64 || rows < 1 || cols <= 0 || cols % 256) return 0;
  return gemv_ws(T, rows, cols).total;
}

int iqk_gemv(const iqk_weights* w, int32_t expert, const float* values, const uint16_t* x, int32_t T, float* y,
             void* workspace, size_t ws_bytes, void* stream) {
  WDev wd;
  Values V;
  int rc;
  if ((rc = check_weights(w, &wd)) || (rc = check_values(values, &V))) return rc;
  if (expert < 0 || expert >= wd.experts || !x || !y) return IQK_EINVAL;
  if (!aligned(x, 16) || !aligned(y, 4)) return IQK_EINVAL;  // x is read in 16-byte groups
  if (T < 1 || T > 64) return IQK_EUNSUPPORTED;
  if ((rc = check_ws(workspace, ws_bytes, gemv_ws(T, wd.rows, wd.cols).total))) return rc;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_gemv(wd, w->fmt, expert, V, x, T, y, (char*)workspace, (cudaStream_t)stream, sms));
}

size_t iqk_moe_workspace_bytes(int32_t mode, int32_t T, int32_t topk, int32_t experts, int32_t hidden,
                               int32_t inter) {
  if (T < 1 || topk < 1 || topk > 16 || experts < 1 || hidden <= 0 || inter <= 0 || hidden % 256 || inter % 256)
    return 0;
  if (mode == 0) {
    if (T > 64 || T * topk > kMaxPairs) return 0;
    return decode_ws(T, topk, experts, hidden, inter).total;
  }
  if (mode == 1) {
    if (T > 65536) return 0;
    return prefill_ws(T, topk, experts, hidden, inter).total;
  }
  return 0;
}

int iqk_moe_workspace_layout(int32_t mode, int32_t T, int32_t topk, int32_t experts, int32_t hidden,
                             int32_t inter, iqk_ws_layout* out) {
  if (!out || iqk_moe_workspace_bytes(mode, T, topk, experts, hidden, inter) == 0) return IQK_EINVAL;
  memset(out, 0, sizeof(*out));
  out->h_rows = T * topk;
  if (mode == 0) {
    const DecodeWs L = decode_ws(T, topk, experts, hidden, inter);
    out->status = (int64_t)L.status;
    out->h = (int64_t)L.hperm;
    out->h_order = -1;
  } else {
    const PrefillWs L = prefill_ws(T, topk, experts, hidden, inter);
    out->status = (int64_t)L.status;
    out->h = (int64_t)L.hs;
    out->h_order = (int64_t)L.perm;
  }
  return IQK_OK;
}

static bool host_locked(const void* ptr) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
    (void)cudaGetLastError();  // an unregistered pointer: not an error of the context
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}

// iqk_moe_decode and iqk_moe_decode_host: the same checks, then the same launch
// (host_io: x, ids, p and y in page-locked host memory).
static int moe_decode(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down, const float* values,
                      const uint16_t* x, int32_t T, const int32_t* ids, const float* p, int32_t topk, uint16_t* y,
                      void* workspace, size_t ws_bytes, void* stream, bool host_io) {
  WDev g, u, d;
  Values V;
  int rc;
  if ((rc = check_moe(gate, up, down, &g, &u, &d)) || (rc = check_values(values, &V))) return rc;
  if (!x || !ids || !p || !y) return IQK_EINVAL;
  if (T == 0) return IQK_OK;
  if (T < 0 || topk < 1 || topk > 16) return IQK_EINVAL;
  if (T > 64 || T * topk > kMaxPairs) return IQK_EUNSUPPORTED;
  if (host_io && (reinterpret_cast<uintptr_t>(x) % 16 || !host_locked(x) || !host_locked(ids) || !host_locked(p) ||
                  !host_locked(y)))
    return IQK_EINVAL;
  if ((rc = check_ws(workspace, ws_bytes, decode_ws(T, topk, g.experts, g.cols, g.rows).total))) return rc;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_moe_decode(g, gate->fmt, u, up->fmt, d, down->fmt, V, x, T, ids, p, topk, y, nullptr, 0,
                                       (char*)workspace, (cudaStream_t)stream, sms, host_io));
}

int iqk_moe_decode(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down, const float* values,
                   const uint16_t* x, int32_t T, const int32_t* ids, const float* p, int32_t topk, uint16_t* y,
                   void* workspace, size_t ws_bytes, void* stream) {
  return moe_decode(gate, up, down, values, x, T, ids, p, topk, y, workspace, ws_bytes, stream, false);
}

int iqk_moe_decode_host(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down, const float* values,
                        const uint16_t* x, int32_t T, const int32_t* ids, const float* p, int32_t topk, uint16_t* y,
                        void* workspace, size_t ws_bytes, void* stream) {
  return moe_decode(gate, up, down, values, x, T, ids, p, topk, y, workspace, ws_bytes, stream, true);
}

int iqk_moe_decode_shard(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                         const float* values, const uint16_t* x, int32_t T, const int32_t* ids, const float* p,
                         int32_t topk, int32_t expert_base, float* y_partial, void* workspace, size_t ws_bytes,
                         void* stream) {
  WDev g, u, d;
  Values V;
  int rc;
  if ((rc = check_moe(gate, up, down, &g, &u, &d)) || (rc = check_values(values, &V))) return rc;
  if (!x || !ids || !p || !y_partial || expert_base < 0) return IQK_EINVAL;
  if (T == 0) return IQK_OK;
  if (T < 0 || topk < 1 || topk > 16) return IQK_EINVAL;
  if (T > 64 || T * topk > kMaxPairs) return IQK_EUNSUPPORTED;
  if ((rc = check_ws(workspace, ws_bytes, decode_ws(T, topk, g.experts, g.cols, g.rows).total))) return rc;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_moe_decode(g, gate->fmt, u, up->fmt, d, down->fmt, V, x, T, ids, p, topk, nullptr,
                                       y_partial, expert_base, (char*)workspace, (cudaStream_t)stream, sms));
}

int iqk_f32_to_bf16(const float* in, uint16_t* out, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!in || !out))) return IQK_EINVAL;
  if (n == 0) return IQK_OK;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_to_bf16(in, out, n, (cudaStream_t)stream, sms));
}

int iqk_moe_prefill(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down, const float* values,
                    const uint16_t* x, int32_t T, const int32_t* ids, const float* p, int32_t topk, uint16_t* y,
                    void* workspace, size_t ws_bytes, void* stream) {
  WDev g, u, d;
  Values V;
  int rc;
  if ((rc = check_moe(gate, up, down, &g, &u, &d)) || (rc = check_values(values, &V))) return rc;
  if (!x || !ids || !p || !y) return IQK_EINVAL;
  if (T == 0) return IQK_OK;
  if (T < 0 || topk < 1 || topk > 16) return IQK_EINVAL;
  if (T > 65536) return IQK_EUNSUPPORTED;
  if (!aligned(x, 16) || !aligned(y, 16)) return IQK_EINVAL;
  if ((rc = check_ws(workspace, ws_bytes, prefill_ws(T, topk, g.experts, g.cols, g.rows).total))) return rc;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_moe_prefill(g, gate->fmt, u, up->fmt, d, down->fmt, V, x, T, ids, p, topk, y, nullptr,
                                        0, (char*)workspace, (cudaStream_t)stream, sms));
}

int iqk_moe_prefill_shard(const iqk_weights* gate, const iqk_weights* up, const iqk_weights* down,
                          const float* values, const uint16_t* x, int32_t T, const int32_t* ids, const float* p,
                          int32_t topk, int32_t expert_base, float* y_partial, void* workspace, size_t ws_bytes,
                          void* stream) {
  WDev g, u, d;
  Values V;
  int rc;
  if ((rc = check_moe(gate, up, down, &g, &u, &d)) || (rc = check_values(values, &V))) return rc;
  if (!x || !ids || !p || !y_partial || expert_base < 0) return IQK_EINVAL;
  if (T == 0) return IQK_OK;
  if (T < 0 || topk < 1 || topk > 16) return IQK_EINVAL;
  if (T > 65536) return IQK_EUNSUPPORTED;
  if (!aligned(x, 16) || !aligned(y_partial, 16)) return IQK_EINVAL;
  if ((rc = check_ws(workspace, ws_bytes, prefill_ws(T, topk, g.experts, g.cols, g.rows).total))) return rc;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_moe_prefill(g, gate->fmt, u, up->fmt, d, down->fmt, V, x, T, ids, p, topk, nullptr,
                                        y_partial, expert_base, (char*)workspace, (cudaStream_t)stream, sms));
}

int iqk_moe_combine(const float* rows, const float* p, int32_t T, int32_t topk, int32_t hidden, uint16_t* y,
                    void* stream) {
  if (T == 0) return IQK_OK;
  if (!rows || !p || !y || T < 0 || topk < 1 || topk > 16) return IQK_EINVAL;
  if (hidden <= 0 || hidden % 4) return IQK_ESHAPE;
  if (!aligned(rows, 16) || !aligned(y, 8)) return IQK_EINVAL;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_combine(rows, p, T, topk, hidden, y, (cudaStream_t)stream, sms));
}

int iqk_moe_status(const void* workspace, void* stream) {
  if (!workspace) return IQK_EINVAL;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  int32_t s = 0;
  e = cudaMemcpy(&s, workspace, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (s & 2) return IQK_ETIMEOUT;
  if (s & 1) return IQK_EINVAL;
  return IQK_OK;
}

size_t iqk_route_workspace_bytes(int32_t T, int32_t topk, int32_t experts) {
  if (T < 1 || topk < 1 || topk > 16 || experts < 1) return 0;
  return align256(16) + align256(route_scratch_ints(T * topk, experts) * 4);
}

int iqk_moe_route(const int32_t* ids, int32_t T, int32_t topk, int32_t experts, int32_t* counts, int32_t* offsets,
                  int32_t* perm, void* workspace, size_t ws_bytes, void* stream) {
  if (!ids || !counts || !offsets || !perm) return IQK_EINVAL;
  if (T < 1 || topk < 1 || topk > 16 || experts < 1) return IQK_EINVAL;
  if (T > 65536 || experts > 50000) return IQK_EUNSUPPORTED;
  int rc;
  if ((rc = check_ws(workspace, ws_bytes, iqk_route_workspace_bytes(T, topk, experts)))) return rc;
  char* ws = (char*)workspace;
  return from_launch(launch_route(ids, T, topk, experts, counts, offsets, perm, reinterpret_cast<int32_t*>(ws),
                                  reinterpret_cast<int32_t*>(ws + align256(16)), (cudaStream_t)stream));
}

int iqk_floor(const iqk_weights* w, const int32_t* expert_list, int32_t n_experts, uint32_t* out, void* stream) {
  WDev wd;
  int rc;
  if ((rc = check_weights(w, &wd))) return rc;
  if (!expert_list || !out || n_experts < 1) return IQK_EINVAL;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(launch_floor(wd, w->fmt, expert_list, n_experts, out, (cudaStream_t)stream, sms));
}

int iqk_floor_status(void* stream) {
  int32_t s = 0;
  if (read_floor_status((cudaStream_t)stream, &s)) return cuda_fail(cudaGetLastError());
  return (s & 2) ? IQK_ETIMEOUT : IQK_OK;
}

int iqk_set_wait_limit_ns(uint64_t limit_ns, int32_t expire) {
  set_wait_limit(limit_ns, expire);
  return IQK_OK;
}

}  // extern "C"

// ------------------------------------------------------------ switch linear
namespace {
// Pair count at or below which the auto mode takes the decode-style kernel.
constexpr int kSwitchDecodeMaxPairs = IQK_SWITCH_DECODE_MAX_PAIRS;

bool switch_decode_ok(int T, int topk) { return T <= 64 && T * topk <= kMaxPairs; }
bool switch_gemm_ok(const WDev& w, int T) { return w.rows % 256 == 0 && T <= 65536; }

int switch_pick(int mode, const WDev& w, int T, int topk) {
  const bool dec = switch_decode_ok(T, topk), gem = switch_gemm_ok(w, T);
  if (mode == 1) return dec ? 1 : -1;
  if (mode == 2) return gem ? 2 : -1;
  if (mode != 0) return -2;
  if (dec && (T * topk <= kSwitchDecodeMaxPairs || !gem)) return 1;
  return gem ? 2 : -1;
}
}  // namespace

extern "C" size_t iqk_switch_linear_workspace_bytes(int32_t mode, int32_t T, int32_t topk, int32_t experts,
                                                    int32_t rows, int32_t cols) {
  if (T < 1 || topk < 1 || topk > 16 || experts < 1 || rows < 1 || cols <= 0 || cols % 256) return 0;
  WDev w = {};
  w.rows = rows;
  w.cols = cols;
  w.experts = experts;
  const int pick = switch_pick(mode, w, T, topk);
  if (pick == 1) return switch_ws(T, topk, experts, rows, cols).total;
  if (pick == 2) return switch_gemm_ws(T, topk, experts, rows, cols);
  return 0;
}

extern "C" int iqk_switch_linear(const iqk_weights* w, const float* values, const uint16_t* x, int32_t T,
                                 const int32_t* ids, int32_t topk, float* y, int32_t mode, void* workspace,
                                 size_t ws_bytes, void* stream) {
  WDev wd;
  Values V;
  int rc;
  if ((rc = check_weights(w, &wd)) || (rc = check_values(values, &V))) return rc;
  if (!x || !ids || !y || !aligned(x, 16) || !aligned(y, 16)) return IQK_EINVAL;
  if (topk < 1 || topk > 16) return IQK_EINVAL;
  if (T == 0) return IQK_OK;
  if (T < 0) return IQK_EINVAL;
  const int pick = switch_pick(mode, wd, T, topk);
  if (pick == -2) return IQK_EINVAL;
  if (pick < 0) return IQK_EUNSUPPORTED;
  const size_t need =
      pick == 1 ? switch_ws(T, topk, wd.experts, wd.rows, wd.cols).total : switch_gemm_ws(T, topk, wd.experts, wd.rows, wd.cols);
  if ((rc = check_ws(workspace, ws_bytes, need))) return rc;
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  if (pick == 1)
    return from_launch(launch_switch_decode(wd, w->fmt, V, x, T, ids, topk, y, (char*)workspace, (cudaStream_t)stream,
                                            sms));
  return from_launch(
      launch_switch_gemm(wd, w->fmt, V, x, T, ids, topk, y, (char*)workspace, (cudaStream_t)stream, sms));
}

// ------------------------------------------------------- no-allocation GEMV
// iqk_gemv_static runs the same launches as iqk_gemv, with its scratch in a
// file-scope device array instead of a caller-provided workspace. The array
// lives in every device context that loads the library; every call looks up
// its address in the current context (cudaGetSymbolAddress), so nothing is
// kept across a device reset. What must start at zero (the tile counters) is
// zeroed by the call's own first kernel. Calls that overlap in time on one
// device share the array and race; the caller serialises them (one stream,
// or events).
namespace {
static __device__ __align__(256) unsigned char g_gemv_scratch[IQK_GEMV_STATIC_SCRATCH_BYTES];
}  // namespace

extern "C" int iqk_gemv_static(const iqk_weights* w, int32_t expert, const float* values, const uint16_t* x,
                               int32_t T, float* y, void* stream) {
  WDev wd;
  Values V;
  int rc;
  if ((rc = check_weights(w, &wd)) || (rc = check_values(values, &V))) return rc;
  if (expert < 0 || expert >= wd.experts || !x || !y) return IQK_EINVAL;
  if (!aligned(x, 16) || !aligned(y, 4)) return IQK_EINVAL;
  if (T < 1 || T > 64) return IQK_EUNSUPPORTED;
  if (gemv_ws(T, wd.rows, wd.cols).total > IQK_GEMV_STATIC_SCRATCH_BYTES) return IQK_EWORKSPACE;
  void* scratch = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&scratch, g_gemv_scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  const int sms = num_sms();
  if (sms < 0) return cuda_fail(cudaGetLastError());
  return from_launch(
      launch_gemv(wd, w->fmt, expert, V, x, T, y, static_cast<char*>(scratch), (cudaStream_t)stream, sms, false));
}
