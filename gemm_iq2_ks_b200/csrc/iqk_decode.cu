// Decode-side kernels: single-expert GEMV, routed gate/up + SwiGLU, routed
// down + weighted combine, and the deleted-decode address floor.
//
// mlx-iqk 0.1.1 PKG-INFO: "a call with few token-expert pairs runs the fused
// decode GEMV" (section "Surface"); reconstruction d*float(scale_index)*
// values[4*alphabet+code] (section "Format"); pricing against "identical
// loads, decode removed" (section "Pricing").
//
// Work is cut into units of 16 weight rows x one k-chunk (nb 256-weight
// blocks). Each warp owns a two-stage ring in shared memory: one elected lane
// stages a unit's qs tile with a 2-D TMA load (no multicast), the warp decodes
// it against a per-CTA table of bf16(scale_index * value) entries with
// byte-permutes and reduces with m16n8k16 tensor-core MMAs (tokens or pairs
// as the MMA's N). Partial sums of a tile's k-chunks meet in the workspace;
// the last unit to finish a tile (device-scope counter) sums them in chunk
// order, so results do not depend on arrival order.
#include <algorithm>

#include "iqk_device.cuh"
#include "iqk_internal.h"

namespace iqk {

Chunking chunking(int rows, int cols) {
  Chunking c;
  const int nbk = cols / 256;
  c.nb = (nbk % 2 == 0) ? 2 : 1;
  c.nkc = nbk / c.nb;
  c.tiles = (rows + kTile - 1) / kTile;
  return c;
}

// ---------------------------------------------------------- unit scales
// A unit's scale planes (16 rows, full reduction width) sit in a per-warp
// shared-memory slot with the global layout of those rows:
//   IQ2_KS: scl [16][nbk] u32 | sch [16][nbk] u8 | sex [16][nbk] u8 | dv [16] u16
//   IQ2_K:  scl [16][2 nbk] u32 | sex [16][nbk] u16 | dv [16][nbk] u16
// (nbk = 256-weight blocks per row). Every part starts on a 16-byte boundary.
template <int FMT>
struct Slot {
  static __host__ __device__ __forceinline__ uint32_t scl_off(int) { return 0; }
  static __host__ __device__ __forceinline__ uint32_t b_off(int nbk) { return FMT == FMT_KS ? 64u * nbk : 128u * nbk; }
  static __host__ __device__ __forceinline__ uint32_t c_off(int nbk) { return FMT == FMT_KS ? 80u * nbk : 160u * nbk; }
  static __host__ __device__ __forceinline__ uint32_t bytes(int nbk) { return FMT == FMT_KS ? 96u * nbk + 32u : 192u * nbk; }
};

template <int F0, int F1>
__host__ __device__ inline uint32_t slot_bytes2(int nbk) {
  const uint32_t a = Slot<F0>::bytes(nbk), b = Slot<F1>::bytes(nbk);
  return a > b ? a : b;
}

// Table indices of the sub-blocks covering words 4t..4t+3 of block kb of row r.
// IQ2_KS: (low4 | high<<4) + 32*alphabet, words (4t, 4t+1) in sub-block 2t.
// IQ2_K:  nibble + 16*alphabet, word 4t+m is sub-block 4t+m.
template <int FMT>
__device__ __forceinline__ void combos_smem(const uint8_t* slot, int nbk, int r, int kb, int t, uint32_t (&c)[4]) {
  if constexpr (FMT == FMT_KS) {
    const uint32_t s = reinterpret_cast<const uint32_t*>(slot)[r * nbk + kb];
    const uint32_t h = slot[Slot<FMT>::b_off(nbk) + r * nbk + kb];
    const uint32_t a = slot[Slot<FMT>::c_off(nbk) + r * nbk + kb];
    const uint32_t sb = (s >> (8 * t)) & 0xFFu;
    const uint32_t hb = (h >> (2 * t)) & 3u;
    const uint32_t ab = (a >> (2 * t)) & 3u;
    const uint32_t c0 = (sb & 15u) | ((hb & 1u) << 4) | ((ab & 1u) << 5);
    const uint32_t c1 = (sb >> 4) | ((hb >> 1) << 4) | ((ab >> 1) << 5);
    c[0] = c0;
    c[1] = c0;
    c[2] = c1;
    c[3] = c1;
  } else {
    const uint32_t sw = reinterpret_cast<const uint32_t*>(slot)[r * 2 * nbk + 2 * kb + (t >> 1)] >> (16 * (t & 1));
    const uint32_t x = (reinterpret_cast<const uint16_t*>(slot + Slot<FMT>::b_off(nbk))[r * nbk + kb] >> (4 * t)) & 15u;
#pragma unroll
    for (int m = 0; m < 4; m++) c[m] = ((sw >> (4 * m)) & 15u) | (((x >> m) & 1u) << 4);
  }
}

// Row scale d: IQ2_KS per row, IQ2_K per (row, block).
template <int FMT>
__device__ __forceinline__ float d_smem(const uint8_t* slot, int nbk, int r, int kb) {
  // IQ2_KS: dv follows the 16 * nbk sex bytes; IQ2_K: dv is the third plane
  const uint16_t* dv =
      reinterpret_cast<const uint16_t*>(slot + Slot<FMT>::c_off(nbk) + (FMT == FMT_KS ? 16u * nbk : 0u));
  return __half2float(__ushort_as_half(FMT == FMT_KS ? dv[r] : dv[r * nbk + kb]));
}

// Entry c of the table: bf16 of scale_index * values[4*alphabet + code] for
// code 0..3, packed two per word (code 0 in the low half).
template <int FMT>
__device__ __forceinline__ void build_lut(uint2* lut, const Values& V) {
  const int n = FMT == FMT_KS ? 64 : 32;
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    int idx, a;
    if (FMT == FMT_KS) {
      idx = (c & 31) - 16;
      a = c >> 5;
    } else {
      idx = (c & 15) - 8;
      a = c >> 4;
    }
    const float fi = (float)idx;
    const float e0 = __fmul_rn(fi, a ? V.v[4] : V.v[0]);
    const float e1 = __fmul_rn(fi, a ? V.v[5] : V.v[1]);
    const float e2 = __fmul_rn(fi, a ? V.v[6] : V.v[2]);
    const float e3 = __fmul_rn(fi, a ? V.v[7] : V.v[3]);
    lut[c] = make_uint2(pack_bf16x2(e0, e1), pack_bf16x2(e2, e3));
  }
}

// One 256-weight block of a 16-row tile: part[m] += W(16 x 64 of word m) * B.
// Each of the block's four qs words feeds its own accumulator set, so
// consecutive MMAs do not wait on each other; half a block's activation
// fragments are requested ahead of their MMAs.
template <int FMT, int NT>
__device__ __forceinline__ void block_mma(const uint32_t* __restrict__ sq, int ldw, int bcol, const uint16_t* const (&src)[NT],
                                          const uint32_t (&cg)[4], const uint32_t (&ch)[4],
                                          const uint2* __restrict__ lut, float (&part)[4][NT][4], int g, int t,
                                          uint32_t k65536) {
  // activation fragments of slots (m, i): 8 bytes each, 32 consecutive bytes per word m
  uint4 bf[NT][4];
#pragma unroll
  for (int n = 0; n < NT; n++)
#pragma unroll
    for (int f = 0; f < 4; f++) bf[n][f] = src[n] ? ld_nc_u4(src[n] + 8 * f) : make_uint4(0u, 0u, 0u, 0u);
  const uint4 qg = *reinterpret_cast<const uint4*>(sq + g * ldw + bcol + 4 * t);
  const uint4 qh = *reinterpret_cast<const uint4*>(sq + (g + 8) * ldw + bcol + 4 * t);
#pragma unroll
  for (int m = 0; m < 4; m++) {
    if (m == 2) {
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int f = 0; f < 4; f++) bf[n][f] = src[n] ? ld_nc_u4(src[n] + 32 + 8 * f) : make_uint4(0u, 0u, 0u, 0u);
    }
    const uint32_t wg = m == 0 ? qg.x : m == 1 ? qg.y : m == 2 ? qg.z : qg.w;
    const uint32_t wh = m == 0 ? qh.x : m == 1 ? qh.y : m == 2 ? qh.z : qh.w;
    const uint2 tg = lut[cg[m]];
    const uint2 th = lut[ch[m]];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const Pair2 pg = lookup_slot_mh(wg, i, tg.x, tg.y, k65536);
      const Pair2 ph = lookup_slot_mh(wh, i, th.x, th.y, k65536);
#pragma unroll
      for (int n = 0; n < NT; n++) {
        const uint4 b4 = bf[n][2 * (m & 1) + (i >> 1)];
        const uint32_t b0 = (i & 1) ? b4.z : b4.x, b1 = (i & 1) ? b4.w : b4.y;
        mma_bf16_4(part[m][n][0], part[m][n][1], part[m][n][2], part[m][n][3], pg.lo, ph.lo, pg.hi, ph.hi, b0, b1);
      }
    }
  }
}

// ---------------------------------------------------------- routing (CTA)
// Distinct experts of a decode call and the pairs routed to each, rebuilt by
// every CTA from the raw ids (at most kMaxPairs pairs).
struct RouteView {
  int32_t* ids;      // [n] expert id or -1 when out of range
  int16_t* sorted;   // [n] valid pair indices ordered by (expert, pair)
  int16_t* ustart;   // [n+1] start of distinct expert u in `sorted`
  int32_t* uexp;     // [n] expert id of u
  uint8_t* first;    // [n] scratch
  int32_t* scalars;  // [0] = D, [1] = valid pairs
};

__host__ __device__ inline size_t route_smem_bytes(int n) {
  return (size_t)n * 4 + (size_t)n * 2 + (size_t)(n + 1) * 2 + (size_t)n * 4 + (size_t)n + 16 + 64;
}

__device__ __forceinline__ RouteView carve_route(uint8_t* p, int n) {
  RouteView r;
  r.ids = reinterpret_cast<int32_t*>(p);
  p += (size_t)n * 4;
  r.uexp = reinterpret_cast<int32_t*>(p);
  p += (size_t)n * 4;
  r.scalars = reinterpret_cast<int32_t*>(p);
  p += 16;
  r.sorted = reinterpret_cast<int16_t*>(p);
  p += (size_t)n * 2;
  r.ustart = reinterpret_cast<int16_t*>(p);
  p += (size_t)(n + 1) * 2;
  r.first = p;
  return r;
}

__device__ __forceinline__ void build_route(const int32_t* __restrict__ ids, int n, int E, RouteView r) {
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int e = ids[p];
    r.ids[p] = (e >= 0 && e < E) ? e : -1;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int ep = r.ids[p];
    if (ep < 0) continue;
    int rank = 0;
    for (int q = 0; q < n; q++) {
      const int eq = r.ids[q];
      rank += (eq >= 0) && (eq < ep || (eq == ep && q < p));
    }
    r.sorted[rank] = (int16_t)p;
  }
  if (threadIdx.x == 0) {
    int v = 0;
    for (int q = 0; q < n; q++) v += r.ids[q] >= 0;
    r.scalars[1] = v;
  }
  __syncthreads();
  const int nv = r.scalars[1];
  for (int k = threadIdx.x; k < nv; k += blockDim.x)
    r.first[k] = (k == 0) || (r.ids[r.sorted[k - 1]] != r.ids[r.sorted[k]]);
  __syncthreads();
  for (int k = threadIdx.x; k < nv; k += blockDim.x) {
    if (!r.first[k]) continue;
    int u = 0;
    for (int q = 0; q < k; q++) u += r.first[q];
    r.uexp[u] = r.ids[r.sorted[k]];
    r.ustart[u] = (int16_t)k;
  }
  if (threadIdx.x == 0) {
    int D = 0;
    for (int q = 0; q < nv; q++) D += r.first[q];
    r.scalars[0] = D;
    r.ustart[D] = (int16_t)nv;
  }
  __syncthreads();
}

// ------------------------------------------------------------- prep kernel
// Slot-transposes the activations (x[t][16w + i + 4j] -> xp[t][16w + 4i + j]),
// zeroes the tile counters and records out-of-range expert ids.
__global__ void __launch_bounds__(256) k_prep(const uint16_t* __restrict__ x, int T, int cols,
                                              uint16_t* __restrict__ xp, int32_t* __restrict__ zero,
                                              int nzero, const int32_t* __restrict__ ids, int npairs, int E,
                                              int32_t* __restrict__ status) {
  griddep_launch();
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int nth = gridDim.x * blockDim.x;
  for (int i = tid; i < nzero; i += nth) zero[i] = 0;
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    int bad = 0;
    for (int p = threadIdx.x; p < npairs; p += 32) bad |= (ids[p] < 0 || ids[p] >= E);
    bad = __any_sync(0xffffffffu, bad);
    if (threadIdx.x == 0) status[0] = bad ? 1 : 0;
  }
  // one thread per 16-element group: out[4i + j] = in[i + 4j]
  const int groups = cols / 16;
  const int n = T * groups;
  for (int gi = tid; gi < n; gi += nth) {
    const int t = gi / groups, grp = gi - t * groups;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * cols + 16 * grp);
    const uint4 a = src[0], b = src[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[8];
#pragma unroll
    for (int i2 = 0; i2 < 4; i2++) {
      const int wa = i2 >> 1;
      const uint32_t sel = (i2 & 1) ? 0x7632u : 0x5410u;
      o[2 * i2] = prmt(w[wa], w[wa + 2], sel);
      o[2 * i2 + 1] = prmt(w[wa + 4], w[wa + 6], sel);
    }
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)t * cols + 16 * grp);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ------------------------------------------------------------ stream kernel
// One kernel for the GEMV-shaped jobs and the floor arm. A unit is 16 rows of
// one matrix over the full reduction width; its columns are the tokens (GEMV)
// or the (token, slot) pairs routed to one distinct expert. Each warp streams
// its units through a ring of kStages chunks (CH 256-weight blocks of the
// unit's qs, by 2-D TMA); a unit's scale planes arrive by 1-D bulk copy into
// one of kStages per-warp slots together with its first chunk, so loads run
// kStages chunks ahead of the decode.
//   GEMV:   y[t][row] = acc (fp32).
//   GATEUP: gate and up units of a tile write partials; the tile's second
//           unit forms h = bf16(silu(g) * u) in the slot-transposed layout.
//   DOWN:   p-weighted partials per (tile, pair); the tile's last unit sums
//           each token's slots in slot order into y (bf16).
//   FLOOR:  identical loads; the decode is replaced by an XOR of every loaded
//           byte into out[expert][row].
enum : int { MODE_GEMV = 0, MODE_GATEUP = 1, MODE_DOWN = 2, MODE_FLOOR = 3 };

struct UnitArgs {
  WDev w0, w1;
  Values V;
  const int32_t* ids;
  const float* p;
  const uint16_t* act;  // slot-transposed activation rows
  int T, topk, expert;
  const int32_t* elist;  // FLOOR: experts to stream
  int nexp;
  float* yf;        // GEMV output [T][rows]
  uint16_t* out16;  // GATEUP: h [pairs][inter]; DOWN: y [T][hidden]
  uint32_t* outx;   // FLOOR: [nexp][rows]
  int32_t* cnt;
  float* part;
  int32_t* status;
  int ch;  // blocks per chunk
};

struct Ring {
  uint32_t* qs;    // [kStages][16][ldw]
  uint8_t* slots;  // [kStages][slot bytes]
  uint64_t* bar;   // [kStages]
};

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Stage the scale planes of rows [row0, row0 + 16) of `w` into `slot`.
// A full tile whose four source ranges all start on 16-byte boundaries is
// bulk-copied (the returned byte count is what the caller expects on the
// barrier; the copies are issued when `issue` is set). Any other tile (past
// the last row, or a shape whose rows do not fall on 16-byte boundaries) is
// filled by the lanes with plain loads, zeros past the last row; that path
// returns 0 and ends with __syncwarp.
template <int FMT>
__device__ __forceinline__ uint32_t stage_scales(uint8_t* slot, const WDev& w, int64_t row0, int valid_rows,
                                                 uint64_t* bar, int lane, bool issue) {
  const int nbk = w.cols / 256;
  const uint32_t b_scl = FMT == FMT_KS ? 64u * nbk : 128u * nbk;  // 16 rows of scl
  const uint32_t b_b = FMT == FMT_KS ? 16u * nbk : 32u * nbk;     // 16 rows of sch (KS) / sex (K)
  const uint32_t b_c = FMT == FMT_KS ? 16u * nbk : 32u * nbk;     // 16 rows of sex (KS) / dv (K)
  const uint8_t* src_scl = reinterpret_cast<const uint8_t*>(w.scl) + row0 * (b_scl / 16);
  const uint8_t* src_b = FMT == FMT_KS ? w.sch + row0 * nbk
                                       : reinterpret_cast<const uint8_t*>(reinterpret_cast<const uint16_t*>(w.sex) + row0 * nbk);
  const uint8_t* src_c = FMT == FMT_KS ? reinterpret_cast<const uint8_t*>(w.sex) + row0 * nbk
                                       : reinterpret_cast<const uint8_t*>(w.dv + row0 * nbk);
  const uint8_t* src_d = reinterpret_cast<const uint8_t*>(w.dv + row0);  // IQ2_KS row scales
  const uintptr_t mis = (reinterpret_cast<uintptr_t>(src_scl) | reinterpret_cast<uintptr_t>(src_b) |
                         reinterpret_cast<uintptr_t>(src_c) | (FMT == FMT_KS ? reinterpret_cast<uintptr_t>(src_d) : 0)) &
                        15u;
  if (valid_rows == kTile && mis == 0) {
    if (issue) {
      bulk_copy(slot, src_scl, b_scl, bar);
      bulk_copy(slot + Slot<FMT>::b_off(nbk), src_b, b_b, bar);
      bulk_copy(slot + Slot<FMT>::c_off(nbk), src_c, b_c, bar);
      if (FMT == FMT_KS) bulk_copy(slot + Slot<FMT>::c_off(nbk) + b_c, src_d, 32u, bar);
    }
    return b_scl + b_b + b_c + (FMT == FMT_KS ? 32u : 0u);
  }
  if (issue) return 0;
  const uint32_t per_scl = b_scl / 16, per_b = b_b / 16, per_c = b_c / 16;  // bytes per row
  for (uint32_t i = lane; i < b_scl / 4; i += 32) {
    const bool ok = (int)(i / (per_scl / 4)) < valid_rows;
    reinterpret_cast<uint32_t*>(slot)[i] = ok ? __ldg(reinterpret_cast<const uint32_t*>(src_scl) + i) : 0u;
  }
  uint8_t* sb = slot + Slot<FMT>::b_off(nbk);
  for (uint32_t i = lane; i < b_b; i += 32) sb[i] = (int)(i / per_b) < valid_rows ? __ldg(src_b + i) : (uint8_t)0;
  uint8_t* sc = slot + Slot<FMT>::c_off(nbk);
  for (uint32_t i = lane; i < b_c; i += 32) sc[i] = (int)(i / per_c) < valid_rows ? __ldg(src_c + i) : (uint8_t)0;
  if (FMT == FMT_KS) {
    uint16_t* sd = reinterpret_cast<uint16_t*>(sc + b_c);
    for (int i = lane; i < kTile; i += 32) sd[i] = i < valid_rows ? __ldg(w.dv + row0 + i) : (uint16_t)0;
  }
  __syncwarp();
  return 0;
}

// Timeout flag of the floor arm, which has no workspace; read with
// cudaMemcpyFromSymbol when diagnosing.
__device__ int32_t g_floor_status;

template <int MODE, int F0, int F1, int NT>
__global__ void __launch_bounds__(kDecodeWarps * 32, NT >= 8 ? 2 : (NT >= 4 ? 3 : 4)) k_stream(const __grid_constant__ CUtensorMap m0,
                                                                 const __grid_constant__ CUtensorMap m1,
                                                                 const __grid_constant__ UnitArgs A) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int K = A.w0.cols, nbk = K / 256;
  const int CH = A.ch, ldw = CH * 16, nch = nbk / CH;
  const int stage_words = kTile * ldw;
  const uint32_t slot_b = slot_bytes2<F0, F1>(nbk);
  const uint32_t k65536 = opaque_u32(65536u);
  constexpr int NC = 8 * NT;
  const int npairs = A.T * A.topk;
  const size_t warp_bytes = (size_t)kStages * (stage_words * 4 + slot_b);
  Ring ring;
  ring.qs = reinterpret_cast<uint32_t*>(smem + wid * warp_bytes);
  ring.slots = smem + wid * warp_bytes + (size_t)kStages * stage_words * 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecodeWarps * warp_bytes);
  ring.bar = bars + wid * kStages;
  uint2* lut0 = reinterpret_cast<uint2*>(bars + kDecodeWarps * kStages);
  uint2* lut1 = lut0 + 64;
  if (MODE != MODE_FLOOR) {
    build_lut<F0>(lut0, A.V);
    if (MODE == MODE_GATEUP) build_lut<F1>(lut1, A.V);
  }
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&ring.bar[s], 1);
    fence_mbar_init();
  }
  RouteView rt{};
  int D = 1;
  if (MODE == MODE_GATEUP || MODE == MODE_DOWN) {
    rt = carve_route(reinterpret_cast<uint8_t*>(lut1 + 64), npairs);
    build_route(A.ids, npairs, A.w0.experts, rt);  // ends with __syncthreads
    D = rt.scalars[0];
  } else {
    if (MODE == MODE_FLOOR) D = A.nexp;
    __syncthreads();
  }
  constexpr int NMAT = MODE == MODE_GATEUP ? 2 : 1;
  const int rows = A.w0.rows;
  const int tiles = (rows + kTile - 1) / kTile;
  const int nunits = D * NMAT * tiles;
  const int W = gridDim.x * kDecodeWarps;
  const int gw = blockIdx.x * kDecodeWarps + wid;
  // unit id -> (u, mat, tile): gate and up of one tile are adjacent
  auto unit_of = [&](int id, int& u, int& mat, int& tile) {
    mat = id % NMAT;
    const int r = id / NMAT;
    tile = r % tiles;
    u = r / tiles;
  };
  auto expert_of = [&](int u) -> int {
    if (MODE == MODE_GEMV) return A.expert;
    if (MODE == MODE_FLOOR) return A.elist[u];
    return rt.uexp[u];
  };
  // issue cursor: unit iteration `iu`, chunk `ic`; chunks are numbered
  // q = iu * nch + ic. The unit's coordinates are decoded once per unit.
  int iu = 0, ic = 0;
  int cu_mat = 0;
  int64_t cu_row0 = 0;
  auto issue_next = [&]() {
    const int id = gw + iu * W;
    if (id >= nunits) return;
    const int q = iu * nch + ic;
    const int s = q % kStages;
    uint32_t bytes = (uint32_t)stage_words * 4;
    if (ic == 0) {
      int u, mat, tile;
      unit_of(id, u, mat, tile);
      const int e = expert_of(u);
      cu_mat = mat;
      cu_row0 = (int64_t)e * rows + (int64_t)tile * kTile;
      const int valid = min(kTile, rows - tile * kTile);
      const WDev& w = mat ? A.w1 : A.w0;
      // bulk-copyable tile: returns the bytes to expect; otherwise the lanes fill the slot now
      uint8_t* slot = ring.slots + (size_t)(iu % kStages) * slot_b;
      bytes += (mat == 0) ? stage_scales<F0>(slot, w, cu_row0, valid, &ring.bar[s], lane, false)
                          : stage_scales<F1>(slot, w, cu_row0, valid, &ring.bar[s], lane, false);
      if (lane == 0) {
        mbar_arrive_expect_tx(&ring.bar[s], bytes);
        if (mat == 0) stage_scales<F0>(slot, w, cu_row0, valid, &ring.bar[s], lane, true);
        else stage_scales<F1>(slot, w, cu_row0, valid, &ring.bar[s], lane, true);
      }
    } else if (lane == 0) {
      mbar_arrive_expect_tx(&ring.bar[s], bytes);
    }
    if (lane == 0)
      tma_load_2d(ring.qs + (size_t)s * stage_words, cu_mat ? &m1 : &m0, ic * ldw, (int)cu_row0, &ring.bar[s]);
    if (++ic == nch) {
      ic = 0;
      iu++;
    }
  };
  for (int s = 0; s < kStages; s++) issue_next();
  if (MODE == MODE_GATEUP) griddep_launch();
  griddep_wait();
  if (MODE == MODE_DOWN && D == 0) {  // every id out of range: the block output is zero
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < A.T * rows; i += gridDim.x * blockDim.x) A.out16[i] = 0;
    return;
  }

  for (int it = 0;; it++) {
    const int id = gw + it * W;
    if (id >= nunits) break;
    int u, mat, tile;
    unit_of(id, u, mat, tile);
    const int e = expert_of(u);
    int p0 = 0, ncols = A.T;
    if (MODE == MODE_GATEUP || MODE == MODE_DOWN) {
      p0 = rt.ustart[u];
      ncols = rt.ustart[u + 1] - p0;
    }
    const uint16_t* bsrc[NT];
#pragma unroll
    for (int n = 0; n < NT; n++) {
      const int col = 8 * n + g;
      const uint16_t* b = nullptr;
      if (MODE != MODE_FLOOR && col < ncols) {
        if (MODE == MODE_GEMV) b = A.act + (size_t)col * K;
        else if (MODE == MODE_GATEUP) b = A.act + (size_t)(rt.sorted[p0 + col] / A.topk) * K;
        else b = A.act + (size_t)rt.sorted[p0 + col] * K;
      }
      bsrc[n] = b;
    }
    const uint8_t* slot = ring.slots + (size_t)(it % kStages) * slot_b;
    const bool fmt0 = (MODE != MODE_GATEUP) || mat == 0;
    float part[4][NT][4];
#pragma unroll
    for (int m = 0; m < 4; m++)
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) part[m][n][q] = 0.f;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) acc[n][q] = 0.f;
    uint32_t xg = 0, xh = 0;  // FLOOR checksums of rows g and g + 8
    for (int j = 0; j < nch; j++) {
      const int q = it * nch + j;
      const int s = q % kStages;
      if (!mbar_wait_bounded(&ring.bar[s], (uint32_t)((q / kStages) & 1))) {
        if (lane == 0) atomicOr(A.status ? A.status : &g_floor_status, 2);
        for (int k = 1; k < kStages; k++) (void)mbar_wait_bounded(&ring.bar[(q + k) % kStages], (uint32_t)(((q + k) / kStages) & 1));
        return;
      }
      const uint32_t* sq = ring.qs + (size_t)s * stage_words;
      if (MODE == MODE_FLOOR) {
        for (int b = 0; b < CH; b++) {
          const uint4 a4 = *reinterpret_cast<const uint4*>(sq + g * ldw + b * 16 + 4 * t);
          const uint4 b4 = *reinterpret_cast<const uint4*>(sq + (g + 8) * ldw + b * 16 + 4 * t);
          xg ^= a4.x ^ a4.y ^ a4.z ^ a4.w;
          xh ^= b4.x ^ b4.y ^ b4.z ^ b4.w;
        }
      } else {
        for (int b = 0; b < CH; b++) {
          const int kb = j * CH + b;
          const uint16_t* src[NT];
#pragma unroll
          for (int n = 0; n < NT; n++) src[n] = bsrc[n] ? bsrc[n] + 256 * kb + 64 * t : nullptr;
          uint32_t cg[4], ch[4];
          if (fmt0) {
            combos_smem<F0>(slot, nbk, g, kb, t, cg);
            combos_smem<F0>(slot, nbk, g + 8, kb, t, ch);
          } else {
            combos_smem<F1>(slot, nbk, g, kb, t, cg);
            combos_smem<F1>(slot, nbk, g + 8, kb, t, ch);
          }
          const bool kfmt = fmt0 ? (F0 == FMT_K) : (F1 == FMT_K);
          if (kfmt) {
#pragma unroll
            for (int m = 0; m < 4; m++)
#pragma unroll
              for (int n = 0; n < NT; n++)
#pragma unroll
                for (int qq = 0; qq < 4; qq++) part[m][n][qq] = 0.f;
          }
          block_mma<F0, NT>(sq, ldw, b * 16, src, cg, ch, fmt0 ? lut0 : lut1, part, g, t, k65536);
          if (kfmt) {  // IQ2_K: d changes every block
            const float dg = fmt0 ? d_smem<F0>(slot, nbk, g, kb) : d_smem<F1>(slot, nbk, g, kb);
            const float dh = fmt0 ? d_smem<F0>(slot, nbk, g + 8, kb) : d_smem<F1>(slot, nbk, g + 8, kb);
#pragma unroll
            for (int n = 0; n < NT; n++) {
              acc[n][0] = fmaf(dg, (part[0][n][0] + part[1][n][0]) + (part[2][n][0] + part[3][n][0]), acc[n][0]);
              acc[n][1] = fmaf(dg, (part[0][n][1] + part[1][n][1]) + (part[2][n][1] + part[3][n][1]), acc[n][1]);
              acc[n][2] = fmaf(dh, (part[0][n][2] + part[1][n][2]) + (part[2][n][2] + part[3][n][2]), acc[n][2]);
              acc[n][3] = fmaf(dh, (part[0][n][3] + part[1][n][3]) + (part[2][n][3] + part[3][n][3]), acc[n][3]);
            }
          }
        }
      }
      __syncwarp();
      issue_next();
    }
    const int rg = tile * kTile + g, rh = rg + 8;
    if (MODE == MODE_FLOOR) {
      // fold the slot's scale bytes for rows g and g + 8 (byte i of a row's
      // stream lands in byte i & 3 of the word)
      const bool ks = F0 == FMT_KS;
      const uint32_t* s32 = reinterpret_cast<const uint32_t*>(slot);
      const int nw = ks ? nbk : 2 * nbk;
      for (int i = t; i < nw; i += 4) {
        xg ^= s32[g * nw + i];
        xh ^= s32[(g + 8) * nw + i];
      }
      const uint8_t* sb = slot + Slot<F0>::b_off(nbk);
      const uint8_t* sc = slot + Slot<F0>::c_off(nbk);
      const int nbb = ks ? nbk : 2 * nbk;  // bytes per row of the second / third plane
      for (int i = t; i < nbb; i += 4) {
        xg ^= (uint32_t)sb[g * nbb + i] << (8 * (i & 3));
        xh ^= (uint32_t)sb[(g + 8) * nbb + i] << (8 * (i & 3));
        xg ^= (uint32_t)sc[g * nbb + i] << (8 * (i & 3));
        xh ^= (uint32_t)sc[(g + 8) * nbb + i] << (8 * (i & 3));
      }
      if (ks && t == 0) {
        const uint16_t* sd = reinterpret_cast<const uint16_t*>(sc + 16u * nbk);
        xg ^= sd[g];
        xh ^= sd[g + 8];
      }
      xg ^= __shfl_xor_sync(0xffffffffu, xg, 1);
      xg ^= __shfl_xor_sync(0xffffffffu, xg, 2);
      xh ^= __shfl_xor_sync(0xffffffffu, xh, 1);
      xh ^= __shfl_xor_sync(0xffffffffu, xh, 2);
      if (t == 0) {
        if (rg < rows) A.outx[(size_t)u * rows + rg] = xg;
        if (rh < rows) A.outx[(size_t)u * rows + rh] = xh;
      }
      continue;
    }
    const bool kfmt = fmt0 ? (F0 == FMT_K) : (F1 == FMT_K);
    if (!kfmt) {
      const float dg = fmt0 ? d_smem<F0>(slot, nbk, g, 0) : d_smem<F1>(slot, nbk, g, 0);
      const float dh = fmt0 ? d_smem<F0>(slot, nbk, g + 8, 0) : d_smem<F1>(slot, nbk, g + 8, 0);
#pragma unroll
      for (int n = 0; n < NT; n++) {
        acc[n][0] = dg * ((part[0][n][0] + part[1][n][0]) + (part[2][n][0] + part[3][n][0]));
        acc[n][1] = dg * ((part[0][n][1] + part[1][n][1]) + (part[2][n][1] + part[3][n][1]));
        acc[n][2] = dh * ((part[0][n][2] + part[1][n][2]) + (part[2][n][2] + part[3][n][2]));
        acc[n][3] = dh * ((part[0][n][3] + part[1][n][3]) + (part[2][n][3] + part[3][n][3]));
      }
    }

    if (MODE == MODE_GEMV) {
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const int col = 8 * n + 2 * t + (q & 1);
          const int row = tile * kTile + g + 8 * (q >> 1);
          if (col < A.T && row < rows) A.yf[(size_t)col * rows + row] = acc[n][q];
        }
    } else if (MODE == MODE_GATEUP) {
      const size_t ut = (size_t)u * tiles + tile;
      float* slotp = A.part + (ut * 2 + mat) * NC * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) slotp[(8 * n + 2 * t + (q & 1)) * kTile + g + 8 * (q >> 1)] = acc[n][q];
      __syncwarp();
      int prev = 0;
      if (lane == 0) {
        __threadfence();
        prev = atomicAdd(A.cnt + ut, 1);
      }
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != 1) continue;
      __threadfence();
      const float* other = A.part + (ut * 2 + (mat ^ 1)) * NC * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const int col = 8 * n + 2 * t + (q & 1);
          const int r = g + 8 * (q >> 1);
          const int f = tile * kTile + r;
          if (col >= ncols || f >= rows) continue;
          const float o = __ldcg(other + col * kTile + r);
          const float gv = mat == 0 ? acc[n][q] : o;
          const float uv = mat == 0 ? o : acc[n][q];
          const float h = gv / (1.0f + __expf(-gv)) * uv;
          A.out16[(size_t)rt.sorted[p0 + col] * rows + perm16(f)] = f32_to_bf16_bits(h);
        }
    } else {
      float* slab = A.part + (size_t)tile * npairs * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const int col = 8 * n + 2 * t + (q & 1);
          if (col >= ncols) continue;
          const int pair = rt.sorted[p0 + col];
          slab[(size_t)pair * kTile + g + 8 * (q >> 1)] = __ldg(A.p + pair) * acc[n][q];
        }
      __syncwarp();
      int prev = 0;
      if (lane == 0) {
        __threadfence();
        prev = atomicAdd(A.cnt + tile, 1);
      }
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != D - 1) continue;
      __threadfence();
      for (int o = lane; o < A.T * kTile; o += 32) {
        const int tok = o / kTile, r = o % kTile;
        const int row = tile * kTile + r;
        if (row >= rows) continue;
        float sum = 0.f;
        for (int jj = 0; jj < A.topk; jj++) {
          const int pair = tok * A.topk + jj;
          if (rt.ids[pair] < 0) continue;
          sum += __ldcg(slab + (size_t)pair * kTile + r);
        }
        A.out16[(size_t)tok * rows + row] = f32_to_bf16_bits(sum);
      }
    }
  }
}

// ================================================================== host

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int make_qs_map(CUtensorMap* map, const WDev& w, int nb) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return -4;
  const cuuint64_t dims[2] = {(cuuint64_t)(w.cols / 16), (cuuint64_t)w.experts * (cuuint64_t)w.rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(w.cols / 16) * 4};
  const cuuint32_t box[2] = {(cuuint32_t)(nb * 16), (cuuint32_t)kTile};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(w.qs), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -4;
}

static int chunk_blocks(int cols) {
  const int nbk = cols / 256;
  return nbk % 2 == 0 ? 2 : 1;
}

template <int F0, int F1>
static size_t stream_smem(int cols, int npairs, bool route) {
  const int nbk = cols / 256, ch = chunk_blocks(cols);
  const size_t warp = (size_t)kStages * ((size_t)kTile * ch * 16 * 4 + slot_bytes2<F0, F1>(nbk));
  return kDecodeWarps * warp + (size_t)kDecodeWarps * kStages * 8 + 2 * 64 * 8 + (route ? route_smem_bytes(npairs) : 0);
}

static int nt_for(int cols_needed) { return cols_needed <= 8 ? 1 : cols_needed <= 16 ? 2 : cols_needed <= 32 ? 4 : 8; }

// Per (kernel, dynamic smem) caches so that a call made during stream
// capture issues no attribute or occupancy queries after the first call.
struct KernelCache {
  const void* fn;
  size_t smem_set;
  size_t occ_smem;
  int occ;
};
static KernelCache g_kcache[256];
static int g_kcache_n = 0;

static KernelCache* kcache(const void* fn) {
  for (int i = 0; i < g_kcache_n; i++)
    if (g_kcache[i].fn == fn) return &g_kcache[i];
  if (g_kcache_n == 256) return nullptr;
  g_kcache[g_kcache_n] = KernelCache{fn, 0, (size_t)-1, 0};
  return &g_kcache[g_kcache_n++];
}

template <typename K>
static int occupancy_grid(K kernel, size_t smem, int units_max, int num_sms) {
  KernelCache* kc = kcache(reinterpret_cast<const void*>(kernel));
  int per_sm = 0;
  if (kc && kc->occ_smem == smem) {
    per_sm = kc->occ;
  } else {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kDecodeWarps * 32, smem) != cudaSuccess)
      return -1;
    if (kc) {
      kc->occ_smem = smem;
      kc->occ = per_sm;
    }
  }
  if (per_sm < 1) return -1;
  per_sm = std::min(per_sm, 4);
  int want = (units_max + kDecodeWarps - 1) / kDecodeWarps;
  return std::max(1, std::min(want, per_sm * num_sms));
}

template <typename K>
static int set_smem(K kernel, size_t smem) {
  KernelCache* kc = kcache(reinterpret_cast<const void*>(kernel));
  if (kc && kc->smem_set >= smem) return 0;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return -4;
  if (kc) kc->smem_set = smem;
  return 0;
}

static cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

GemvWs gemv_ws(int T, int rows, int cols) {
  GemvWs ws;
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.xperm = o;
  o = align256(o + (size_t)T * cols * 2);
  ws.cnt = o;
  ws.part = o;
  ws.total = o;
  return ws;
}

template <int MODE, int F0, int F1, int NT>
static int launch_stream(const CUtensorMap& m0, const CUtensorMap& m1, const UnitArgs& a, int units_max,
                         cudaStream_t st, int num_sms, bool pdl) {
  auto kern = k_stream<MODE, F0, F1, NT>;
  const size_t smem = stream_smem<F0, F1>(a.w0.cols, a.T * a.topk, MODE == MODE_GATEUP || MODE == MODE_DOWN);
  if (set_smem(kern, smem)) return -4;
  const int grid = occupancy_grid(kern, smem, units_max, num_sms);
  if (grid < 0) return -4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1] = {pdl_attr()};
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, m0, m1, a) == cudaSuccess ? 0 : -4;
}

template <int FMT, int NT>
static int gemv_impl(const WDev& w, int expert, const Values& V, const uint16_t* x, int T, float* y, char* ws,
                     cudaStream_t st, int num_sms) {
  const int ch = chunk_blocks(w.cols);
  const GemvWs L = gemv_ws(T, w.rows, w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, ch)) return -4;
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * (w.cols / 16) + 63) / 64)));
  k_prep<<<pblocks, 256, 0, st>>>(x, T, w.cols, xp, nullptr, 0, nullptr, 0, 1, status);
  if (cudaGetLastError() != cudaSuccess) return -4;
  UnitArgs a = {};
  a.w0 = w;
  a.w1 = w;
  a.V = V;
  a.act = xp;
  a.T = T;
  a.topk = 1;
  a.expert = expert;
  a.yf = y;
  a.status = status;
  a.ch = ch;
  return launch_stream<MODE_GEMV, FMT, FMT, NT>(map, map, a, (w.rows + kTile - 1) / kTile, st, num_sms, true);
}

int launch_gemv(const WDev& w, int fmt, int expert, const Values& V, const uint16_t* x, int T, float* y, char* ws,
                cudaStream_t st, int num_sms) {
  const int NT = nt_for(T);
#define IQK_GEMV(F, N) \
  if (fmt == F && NT == N) return gemv_impl<F, N>(w, expert, V, x, T, y, ws, st, num_sms);
  IQK_GEMV(FMT_KS, 1) IQK_GEMV(FMT_KS, 2) IQK_GEMV(FMT_KS, 4) IQK_GEMV(FMT_KS, 8)
  IQK_GEMV(FMT_K, 1) IQK_GEMV(FMT_K, 2) IQK_GEMV(FMT_K, 4) IQK_GEMV(FMT_K, 8)
#undef IQK_GEMV
  return -3;
}

DecodeWs decode_ws(int T, int topk, int experts, int hidden, int inter) {
  DecodeWs ws;
  const int npairs = T * topk;
  ws.dmax = std::min(npairs, experts);
  ws.nt = nt_for(T);
  ws.nc = 8 * ws.nt;
  ws.c2 = chunking(inter, hidden);
  ws.c3 = chunking(hidden, inter);
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.xperm = o;
  o = align256(o + (size_t)T * hidden * 2);
  ws.hperm = o;
  o = align256(o + (size_t)npairs * inter * 2);
  ws.cnt2 = o;
  o = align256(o + (size_t)ws.dmax * ws.c2.tiles * 4);
  ws.cnt3 = o;
  o = align256(o + (size_t)ws.c3.tiles * 4);
  ws.part2 = o;
  o = align256(o + (size_t)ws.dmax * ws.c2.tiles * 2 * ws.nc * kTile * 4);
  ws.part3 = o;
  o = align256(o + (size_t)ws.c3.tiles * npairs * kTile * 4);
  ws.total = o;
  return ws;
}

template <int FG, int FU, int FD, int NT>
static int decode_impl(const WDev& g, const WDev& u, const WDev& d, const Values& V, const uint16_t* x, int T,
                       const int32_t* ids, const float* p, int topk, uint16_t* y, char* ws, cudaStream_t st,
                       int num_sms) {
  const DecodeWs L = decode_ws(T, topk, g.experts, g.cols, g.rows);
  const int npairs = T * topk;
  const int ch2 = chunk_blocks(g.cols), ch3 = chunk_blocks(d.cols);
  CUtensorMap mg, mu, md;
  if (make_qs_map(&mg, g, ch2) || make_qs_map(&mu, u, ch2) || make_qs_map(&md, d, ch3)) return -4;
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  uint16_t* hp = reinterpret_cast<uint16_t*>(ws + L.hperm);
  int32_t* cnt2 = reinterpret_cast<int32_t*>(ws + L.cnt2);
  int32_t* cnt3 = reinterpret_cast<int32_t*>(ws + L.cnt3);
  const int nzero = (int)((L.part2 - L.cnt2) / 4);  // both counter arrays
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * (g.cols / 16) + 63) / 64)));
  k_prep<<<pblocks, 256, 0, st>>>(x, T, g.cols, xp, cnt2, nzero, ids, npairs, g.experts, status);
  if (cudaGetLastError() != cudaSuccess) return -4;
  UnitArgs a = {};
  a.w0 = g;
  a.w1 = u;
  a.V = V;
  a.ids = ids;
  a.p = p;
  a.act = xp;
  a.T = T;
  a.topk = topk;
  a.out16 = hp;
  a.cnt = cnt2;
  a.part = reinterpret_cast<float*>(ws + L.part2);
  a.status = status;
  a.ch = ch2;
  int rc = launch_stream<MODE_GATEUP, FG, FU, NT>(mg, mu, a, L.dmax * 2 * L.c2.tiles, st, num_sms, true);
  if (rc) return rc;
  UnitArgs b = a;
  b.w0 = d;
  b.w1 = d;
  b.act = hp;
  b.out16 = y;
  b.cnt = cnt3;
  b.part = reinterpret_cast<float*>(ws + L.part3);
  b.ch = ch3;
  return launch_stream<MODE_DOWN, FD, FD, NT>(md, md, b, L.dmax * L.c3.tiles, st, num_sms, true);
}

int launch_moe_decode(const WDev& g, int fg, const WDev& u, int fu, const WDev& d, int fd, const Values& V,
                      const uint16_t* x, int T, const int32_t* ids, const float* p, int topk, uint16_t* y, char* ws,
                      cudaStream_t st, int num_sms) {
  const int NT = nt_for(T);
  const int key = fg * 4 + fu * 2 + fd;
#define IQK_DEC(G, U, D, N)                  \
  if (key == G * 4 + U * 2 + D && NT == N) \
    return decode_impl<G, U, D, N>(g, u, d, V, x, T, ids, p, topk, y, ws, st, num_sms);
#define IQK_DEC_N(G, U, D) IQK_DEC(G, U, D, 1) IQK_DEC(G, U, D, 2) IQK_DEC(G, U, D, 4) IQK_DEC(G, U, D, 8)
  IQK_DEC_N(0, 0, 0) IQK_DEC_N(0, 0, 1) IQK_DEC_N(0, 1, 0) IQK_DEC_N(0, 1, 1)
  IQK_DEC_N(1, 0, 0) IQK_DEC_N(1, 0, 1) IQK_DEC_N(1, 1, 0) IQK_DEC_N(1, 1, 1)
#undef IQK_DEC_N
#undef IQK_DEC
  return -3;
}

int launch_floor(const WDev& w, int fmt, const int32_t* experts, int n, uint32_t* out, cudaStream_t st,
                 int num_sms) {
  const int ch = chunk_blocks(w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, ch)) return -4;
  UnitArgs a = {};
  a.w0 = w;
  a.w1 = w;
  a.elist = experts;
  a.nexp = n;
  a.outx = out;
  a.T = 1;
  a.topk = 1;
  a.ch = ch;
  a.status = nullptr;  // the floor reports a timeout through g_floor_status
  const int units = n * ((w.rows + kTile - 1) / kTile);
  if (fmt == FMT_KS) return launch_stream<MODE_FLOOR, FMT_KS, FMT_KS, 1>(map, map, a, units, st, num_sms, false);
  return launch_stream<MODE_FLOOR, FMT_K, FMT_K, 1>(map, map, a, units, st, num_sms, false);
}

}  // namespace iqk
