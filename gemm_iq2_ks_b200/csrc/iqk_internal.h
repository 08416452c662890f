// Internal interface between the C-ABI layer (iqk_api.cu) and the kernel
// translation units. Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "iqk_device.cuh"

namespace iqk {

// ---------------------------------------------------------------- dequant
// floor: the same loads and stores with the decode deleted (integer signature).
int launch_dequant(const WDev& w, int fmt, int expert, const Values& V, void* out, bool bf16, bool floor,
                   cudaStream_t st, int num_sms);

// ------------------------------------------------------- decode (GEMV-type)
// Item geometry shared by the GEMV-shaped kernels: 16-row tiles, each item a
// run of `nb` 256-weight blocks of one tile (a slice of the reduction width),
// `nkc` slices per row.
struct Chunking {
  int nb;     // blocks per item (1, 2 or 4)
  int nkc;    // slices per row = blocks_per_row / nb
  int tiles;  // ceil(rows / 16)
};
Chunking chunking(int rows, int cols);
int item_blocks(int cols);

constexpr int kTile = 16;
#ifndef IQK_DECODE_WARPS
#define IQK_DECODE_WARPS 8
#endif
#ifndef IQK_DECODE_STAGES
#define IQK_DECODE_STAGES 2
#endif
constexpr int kDecodeWarps = IQK_DECODE_WARPS;  // warps per decode CTA, each with its own ring
constexpr int kStages = IQK_DECODE_STAGES;      // ring stages per warp, one item each
// Resident CTAs per SM the decode kernels are compiled for (16 warps per SM
// with one or two MMA column groups, 8 with more).
constexpr int kDecodeMinBlocks(int nt) {
  return nt >= 4 ? (8 / kDecodeWarps > 0 ? 8 / kDecodeWarps : 1) : (16 / kDecodeWarps > 0 ? 16 / kDecodeWarps : 1);
}
constexpr int kMaxPairs = 1024;  // routed decode and switch: T * topk

// n / d for 0 <= n < 2^31 as (umulhi(n, m) + n) >> s, with m and s fixed on
// the host (division by an invariant integer, Granlund and Montgomery 1994).
struct FastDiv {
  uint32_t m, s;
  static FastDiv of(uint32_t d) {
    FastDiv f{0u, 0u};
    if (d > 1) {
      uint32_t l = 0;
      while ((1ull << l) < d) l++;
      f.m = (uint32_t)((((1ull << 32) * ((1ull << l) - d)) / d) + 1);
      f.s = l;
    }
    return f;
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
};

// Workspace carve-up for iqk_gemv.
struct GemvWs {
  size_t status, xperm, cnt, part, total;
};
GemvWs gemv_ws(int T, int rows, int cols);

// Workspace carve-up for iqk_moe_decode: status word, transposed x (read
// through L1 when it does not fit shared memory), h, and one counter per run
// of pairs (gate/up tile groups of h written so far).
struct DecodeWs {
  size_t status, xperm, hperm, ready, hin, total;
  Chunking c2, c3;
};
DecodeWs decode_ws(int T, int topk, int experts, int hidden, int inter);

// Host-side TMA descriptor for a qs plane ([experts*rows][cols/16] uint32),
// box [16 rows][nb*16 words]. Returns 0 on success.
int make_qs_map(CUtensorMap* map, const WDev& w, int nb);

// tiles_ok: a tall matrix with few tokens may take the tile kernel (one
// launch); otherwise the prep and stream kernels.
int launch_gemv(const WDev& w, int fmt, int expert, const Values& V, const uint16_t* x, int T,
                float* y, char* ws, cudaStream_t st, int num_sms, bool tiles_ok = true);

// yf non-null: an expert-parallel shard holding experts [ebase, ebase + E)
// writes its float32 partial to yf (y unused) and skips other ids silently.
// host_io: x, ids, p and y are page-locked host memory; the prep kernel
// copies the inputs into the workspace and the down kernel writes y there.
int launch_moe_decode(const WDev& g, int fg, const WDev& u, int fu, const WDev& d, int fd,
                      const Values& V, const uint16_t* x, int T, const int32_t* ids, const float* p,
                      int topk, uint16_t* y, float* yf, int ebase, char* ws, cudaStream_t st, int num_sms,
                      bool host_io = false);
int launch_to_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t st, int num_sms);

// Routed single projection (switch linear), per (token, slot) pair, fp32.
struct SwitchWs {
  size_t status, xperm, total;
};
SwitchWs switch_ws(int T, int topk, int experts, int rows, int cols);
int launch_switch_decode(const WDev& w, int fmt, const Values& V, const uint16_t* x, int T, const int32_t* ids,
                         int topk, float* y, char* ws, cudaStream_t st, int num_sms);
// Grouped-GEMM form (rows a multiple of 256); workspace from switch_gemm_ws.
size_t switch_gemm_ws(int T, int topk, int experts, int rows, int cols);
int launch_switch_gemm(const WDev& w, int fmt, const Values& V, const uint16_t* x, int T, const int32_t* ids,
                       int topk, float* y, char* ws, cudaStream_t st, int num_sms);

// Scale-slot images of w (iqk_pack_slots): their size, and the packing kernel.
size_t slots_bytes(const WDev& w, int fmt);
int launch_pack_slots(const WDev& w, int fmt, uint8_t* out, cudaStream_t st, int num_sms);
int launch_floor(const WDev& w, int fmt, const int32_t* experts, int n, uint32_t* out, cudaStream_t st,
                 int num_sms);
// The floor's timeout flag (cleared by every floor call), after syncing `st`.
int read_floor_status(cudaStream_t st, int32_t* out);

// Bound of the decode-side kernels' data-barrier waits in ns (0: the
// default), and the expire hook (warp 0 of every CTA also waits on a barrier
// nothing arrives on), applied to launches made from now on.
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
void set_wait_limit(uint64_t ns, int expire);

// ----------------------------------------------------------------- prefill
struct PrefillWs {
  size_t status, counts, offsets, perm, tiles, xs, hs, outp, total;
  int npairs, max_tiles;
};
PrefillWs prefill_ws(int T, int topk, int experts, int hidden, int inter);

// Grouping step. `cc` is scratch of route_scratch_ints(T*topk, experts) ints.
// ebase / silent: an expert-parallel shard groups only ids in [ebase, ebase +
// experts), as ids - ebase, and skips the others without flagging them.
int launch_route(const int32_t* ids, int T, int topk, int experts, int32_t* counts, int32_t* offsets,
                 int32_t* perm, int32_t* status, int32_t* cc, cudaStream_t st, int ebase = 0, bool silent = false);
inline size_t route_scratch_ints(int npairs, int experts) {
  return (size_t)((npairs + 1023) / 1024) * experts;
}

// yf non-null: an expert-parallel shard holding experts [ebase, ebase + E)
// writes its float32 partial to yf (y unused) and skips other ids silently.
int launch_moe_prefill(const WDev& g, int fg, const WDev& u, int fu, const WDev& d, int fd,
                       const Values& V, const uint16_t* x, int T, const int32_t* ids, const float* p,
                       int topk, uint16_t* y, float* yf, int ebase, char* ws, cudaStream_t st, int num_sms);
// y[t] = bf16_rn(sum over slots j in order of p[t][j] * rows[t * topk + j]).
// The prefill producer's A operand of rows [row0, row0 + nrows) of one expert, in k order.
int launch_pf_a_tile(const WDev& w, int fmt, int expert, int row0, int nrows, const Values& V, uint16_t* out,
                     cudaStream_t st);
int launch_combine(const float* rows, const float* p, int T, int topk, int H, uint16_t* y, cudaStream_t st,
                   int num_sms);

// Driver entry point for cuTensorMapEncodeTiled (resolved once).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace iqk
