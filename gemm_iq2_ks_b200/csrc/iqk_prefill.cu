// Prefill path (grouped tensor-core GEMMs over experts).
#include "iqk_device.cuh"
#include "iqk_internal.h"

namespace iqk {

PrefillWs prefill_ws(int T, int topk, int experts, int hidden, int inter) {
  PrefillWs ws = {};
  ws.npairs = T * topk;
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.total = o;
  return ws;
}

int launch_moe_prefill(const WDev&, int, const WDev&, int, const WDev&, int, const Values&, const uint16_t*, int,
                       const int32_t*, const float*, int, uint16_t*, char*, cudaStream_t, int) {
  return -3;
}

}  // namespace iqk
