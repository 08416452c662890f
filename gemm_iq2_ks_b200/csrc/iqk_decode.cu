// Decode-side kernels: single-expert GEMV, routed gate/up + SwiGLU, routed
// down + weighted combine (whole block or one expert-parallel shard), the
// routed single projection (switch linear), and the deleted-decode address
// floor.
//
// mlx-iqk 0.1.1 PKG-INFO: "a call with few token-expert pairs runs the fused
// decode GEMV" (section "Surface"); reconstruction d*float(scale_index)*
// values[4*alphabet+code] (section "Format"); pricing against "identical
// loads, decode removed" (section "Pricing").
//
// Work is cut into items of 16 weight rows x `bpi` 256-weight blocks (a
// slice of the reduction width). Each warp owns a ring of item stages in
// shared memory: one elected lane loads an item's qs tile with a 2-D TMA
// (no multicast) while the lanes copy the item's scale slice with cp.async
// onto the same mbarrier; the warp decodes the tile against a per-CTA table
// of bf16(scale_index * value) entries with byte-permutes and reduces with
// m16n8k16 tensor-core MMAs (tokens or pairs as the MMA's N). In the tile
// kernel (routed calls) a CTA takes a group of items and sums their slices in
// shared memory in warp order; in the stream kernel (GEMV, floor) the slices
// of a tile meet in the workspace and the last item to finish a tile
// (device-scope counter) sums them in slice order. Either way results do not
// depend on arrival order.
#include <algorithm>
#include <atomic>

#include "iqk_device.cuh"
#include "iqk_internal.h"

// Selector arithmetic of the code lookup: 0 all shifts on the integer-logic
// pipe (the default: fastest measured on B200 with the unrolled item loop);
// 1 the high-half selector by multiply-high; 2 as 1, plus slot 2's pre-shift
// by multiply-high (moves work from the integer-logic pipe to the FMA pipe).
#ifndef IQK_LOOKUP
#define IQK_LOOKUP 0
#endif

namespace iqk {

// Blocks per item: four for rows of at least 16 blocks, two for shorter rows
// with a multiple of four blocks (more items to spread over the warps), else
// two or one. With a multiple of four blocks per row every scale slice lies
// on the boundaries cp.async needs.
int item_blocks(int cols) {
  const int nbk = cols / 256;
  if (nbk % 4 == 0) return nbk >= 16 ? 4 : 2;
  return nbk % 2 == 0 ? 2 : 1;
}
static bool async_scales(int cols) { return (cols / 256) % 4 == 0; }

Chunking chunking(int rows, int cols) {
  Chunking c;
  const int nbk = cols / 256;
  c.nb = item_blocks(cols);
  c.nkc = nbk / c.nb;
  c.tiles = (rows + kTile - 1) / kTile;
  return c;
}

// ---------------------------------------------------------- item scales
// An item's scale slice (16 rows x bpi blocks) sits in a per-stage slot:
//   IQ2_KS: scl [16][bpi] u32 | sch [16][4] u8 | sex [16][4] u8 | dv [16] u16
//   IQ2_K:  scl [16][2 bpi] u32 | sex [16][bpi] u16 | dv [16][bpi] u16
// Every part starts on a 16-byte boundary (bpi = 1, 2 or 4). An IQ2_KS row of
// sch / sex holds the aligned 4-byte window around the slice's bpi bytes
// (cp.async copies 4 bytes at least); the slice starts `o` bytes into it.
template <int FMT>
struct Slot {
  static __host__ __device__ __forceinline__ uint32_t b_off(int bpi) { return FMT == FMT_KS ? 64u * bpi : 128u * bpi; }
  static __host__ __device__ __forceinline__ uint32_t c_off(int bpi) { return FMT == FMT_KS ? 64u * bpi + 64u : 160u * bpi; }
  static __host__ __device__ __forceinline__ uint32_t dv_off(int bpi) { return 64u * bpi + 128u; }  // IQ2_KS
  static __host__ __device__ __forceinline__ uint32_t bytes(int bpi) { return FMT == FMT_KS ? 64u * bpi + 160u : 192u * bpi; }
};

// IQ2_KS row scale of slot row r (zero past the tile's last row).
__device__ __forceinline__ float d_smem_ks(const uint8_t* slot, int bpi, int r) {
  return __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(slot + Slot<FMT_KS>::dv_off(bpi))[r]));
}

// Bytes between consecutive slots: the larger format's slot, rounded up to
// 128 so that every ring stage and slot keeps a 128-byte aligned base.
template <int F0, int F1>
__host__ __device__ inline uint32_t slot_bytes2(int bpi) {
  const uint32_t a = Slot<F0>::bytes(bpi), b = Slot<F1>::bytes(bpi);
  return ((a > b ? a : b) + 127u) & ~127u;
}

// Table indices of the sub-blocks covering words 4t..4t+3 of slot block lb of row r.
// IQ2_KS: (low4 | high<<4) + 32*alphabet, words (4t, 4t+1) in sub-block 2t.
// IQ2_K:  nibble + 16*alphabet, word 4t+m is sub-block 4t+m.
template <int FMT>
__device__ __forceinline__ void combos_smem(const uint8_t* slot, int bpi, int o, int r, int lb, int t, uint32_t (&c)[4]) {
  if constexpr (FMT == FMT_KS) {
    const uint32_t sb = slot[(r * bpi + lb) * 4 + t];
    const uint32_t h = slot[Slot<FMT>::b_off(bpi) + r * 4 + o + lb];
    const uint32_t a = slot[Slot<FMT>::c_off(bpi) + r * 4 + o + lb];
    const uint32_t hb = (h >> (2 * t)) & 3u;
    const uint32_t ab = (a >> (2 * t)) & 3u;
    const uint32_t c0 = (sb & 15u) | ((hb & 1u) << 4) | ((ab & 1u) << 5);
    const uint32_t c1 = (sb >> 4) | ((hb >> 1) << 4) | ((ab >> 1) << 5);
    c[0] = c0;
    c[1] = c0;
    c[2] = c1;
    c[3] = c1;
  } else {
    const uint32_t sw = reinterpret_cast<const uint16_t*>(slot)[(r * 2 * bpi + 2 * lb) * 2 + t];
    const uint32_t x = (reinterpret_cast<const uint16_t*>(slot + Slot<FMT>::b_off(bpi))[r * bpi + lb] >> (4 * t)) & 15u;
#pragma unroll
    for (int m = 0; m < 4; m++) c[m] = ((sw >> (4 * m)) & 15u) | (((x >> m) & 1u) << 4);
  }
}

// IQ2_K scale d of (row r, slot block lb).
__device__ __forceinline__ float d_smem_k(const uint8_t* slot, int bpi, int r, int lb) {
  const uint16_t* dv = reinterpret_cast<const uint16_t*>(slot + Slot<FMT_K>::c_off(bpi));
  return __half2float(__ushort_as_half(dv[r * bpi + lb]));
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

// 16-byte activation fragment: from shared memory (BSM) or from the
// workspace rows the preceding kernel wrote (a plain load, after the wait).
template <bool BSM>
__device__ __forceinline__ uint4 ld_act(const uint16_t* p) {
  if constexpr (BSM) {
    uint4 r;
    asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(smem_u32(p)));
    return r;
  } else {
    return ld_u4(p);
  }
}

__device__ __forceinline__ Pair2 lookup(uint32_t q, int i, uint32_t t0, uint32_t t1, uint32_t k65536) {
#if IQK_LOOKUP == 0
  (void)k65536;
  return lookup_slot(q, i, t0, t1);
#elif IQK_LOOKUP == 1
  return lookup_slot_mh(q, i, t0, t1, k65536);
#else
  // 2^28 = 65536 << 12, kept opaque through k65536
  if (i == 2) return lookup_slot_mh2(q, t0, t1, k65536, k65536 << 12);
  return lookup_slot_mh(q, i, t0, t1, k65536);
#endif
}

// One 256-weight block of a 16-row tile: part[m] += W(16 x 64 of word m) * B.
// Each of the block's four qs words feeds its own accumulator set, so
// consecutive MMAs do not wait on each other; half a block's activation
// fragments are requested ahead of their MMAs.
template <int FMT, int NT, bool BSM>
__device__ __forceinline__ void block_mma(const uint32_t* __restrict__ sq, int ldw, int bcol, const uint16_t* const (&src)[NT],
                                          const uint32_t (&cg)[4], const uint32_t (&ch)[4],
                                          const uint2* __restrict__ lut, float (&part)[4][NT][4], int g, int t,
                                          uint32_t k65536) {
  // activation fragments of slots (m, i): 8 bytes each, 32 consecutive bytes per word m
  uint4 bf[NT][4];
#pragma unroll
  for (int n = 0; n < NT; n++)
#pragma unroll
    for (int f = 0; f < 4; f++) bf[n][f] = ld_act<BSM>(src[n] + 8 * f);
  const uint4 qg = *reinterpret_cast<const uint4*>(sq + g * ldw + bcol + 4 * t);
  const uint4 qh = *reinterpret_cast<const uint4*>(sq + (g + 8) * ldw + bcol + 4 * t);
#pragma unroll
  for (int m = 0; m < 4; m++) {
    if (m == 2) {
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int f = 0; f < 4; f++) bf[n][f] = ld_act<BSM>(src[n] + 32 + 8 * f);
    }
    const uint32_t wg = m == 0 ? qg.x : m == 1 ? qg.y : m == 2 ? qg.z : qg.w;
    const uint32_t wh = m == 0 ? qh.x : m == 1 ? qh.y : m == 2 ? qh.z : qh.w;
    const uint2 tg = lut[cg[m]];
    const uint2 th = lut[ch[m]];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const Pair2 pg = lookup(wg, i, tg.x, tg.y, k65536);
      const Pair2 ph = lookup(wh, i, th.x, th.y, k65536);
#pragma unroll
      for (int n = 0; n < NT; n++) {
        const uint4 b4 = bf[n][2 * (m & 1) + (i >> 1)];
        const uint32_t b0 = (i & 1) ? b4.z : b4.x, b1 = (i & 1) ? b4.w : b4.y;
        mma_bf16_4(part[m][n][0], part[m][n][1], part[m][n][2], part[m][n][3], pg.lo, ph.lo, pg.hi, ph.hi, b0, b1);
      }
    }
  }
}

// One item (16 rows x bpi blocks) of a matrix in format F0 (fmt0) or F1:
// acc[n] = d * sum over the item's blocks of W * B, rows g and g + 8.
template <int F0, int F1, int NT, bool BSM, int BPI = 0>
__device__ __forceinline__ void item_mma(const uint32_t* sq, const uint8_t* slot, int bpi_rt, int o, int ldw_rt,
                                         const uint16_t* const (&bsrc)[NT], bool fmt0, bool kfmt, const uint2* lut0,
                                         const uint2* lut1, float dg, float dh, int g, int t, uint32_t k65536,
                                         float (&acc)[NT][4]) {
  constexpr int BLKE = BSM ? 320 : 256;  // elements between consecutive 256-weight blocks
  // a compile-time block count (BPI > 0) lets the compiler interleave the blocks
  const int bpi = BPI > 0 ? BPI : bpi_rt;
  const int ldw = BPI > 0 ? 16 * BPI : ldw_rt;
  float part[4][NT][4];
#pragma unroll
  for (int m = 0; m < 4; m++)
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) part[m][n][q] = 0.f;
#pragma unroll
  for (int b = 0; b < (BPI > 0 ? BPI : bpi); b++) {
    const uint16_t* src[NT];
#pragma unroll
    for (int n = 0; n < NT; n++) {
      src[n] = bsrc[n] + BLKE * b;
      if (!BSM && b + 1 < bpi) prefetch_l1(src[n] + BLKE);
    }
    uint32_t cg[4], ch[4];
    if (fmt0) {
      combos_smem<F0>(slot, bpi, o, g, b, t, cg);
      combos_smem<F0>(slot, bpi, o, g + 8, b, t, ch);
    } else {
      combos_smem<F1>(slot, bpi, o, g, b, t, cg);
      combos_smem<F1>(slot, bpi, o, g + 8, b, t, ch);
    }
    if (kfmt) {
#pragma unroll
      for (int m = 0; m < 4; m++)
#pragma unroll
        for (int n = 0; n < NT; n++)
#pragma unroll
          for (int q = 0; q < 4; q++) part[m][n][q] = 0.f;
    }
    block_mma<F0, NT, BSM>(sq, ldw, b * 16, src, cg, ch, fmt0 ? lut0 : lut1, part, g, t, k65536);
    if (kfmt) {  // IQ2_K: d changes every block
      const float kdg = d_smem_k(slot, bpi, g, b);
      const float kdh = d_smem_k(slot, bpi, g + 8, b);
#pragma unroll
      for (int n = 0; n < NT; n++) {
        acc[n][0] = fmaf(kdg, (part[0][n][0] + part[1][n][0]) + (part[2][n][0] + part[3][n][0]), acc[n][0]);
        acc[n][1] = fmaf(kdg, (part[0][n][1] + part[1][n][1]) + (part[2][n][1] + part[3][n][1]), acc[n][1]);
        acc[n][2] = fmaf(kdh, (part[0][n][2] + part[1][n][2]) + (part[2][n][2] + part[3][n][2]), acc[n][2]);
        acc[n][3] = fmaf(kdh, (part[0][n][3] + part[1][n][3]) + (part[2][n][3] + part[3][n][3]), acc[n][3]);
      }
    }
  }
  if (!kfmt) {
#pragma unroll
    for (int n = 0; n < NT; n++) {
      acc[n][0] = dg * ((part[0][n][0] + part[1][n][0]) + (part[2][n][0] + part[3][n][0]));
      acc[n][1] = dg * ((part[0][n][1] + part[1][n][1]) + (part[2][n][1] + part[3][n][1]));
      acc[n][2] = dh * ((part[0][n][2] + part[1][n][2]) + (part[2][n][2] + part[3][n][2]));
      acc[n][3] = dh * ((part[0][n][3] + part[1][n][3]) + (part[2][n][3] + part[3][n][3]));
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
  float* pw;         // [n] routing weights (down kernel)
};

__host__ __device__ inline size_t route_smem_bytes(int n) {
  return (size_t)n * 4 + (size_t)n * 2 + (size_t)(n + 1) * 2 + (size_t)n * 4 + (size_t)n + 16 + 64 + (size_t)n * 4;
}

__device__ __forceinline__ RouteView carve_route(uint8_t* p, int n) {
  RouteView r;
  r.pw = reinterpret_cast<float*>(p);
  p += (size_t)n * 4;
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

// Distinct-expert list of a call. With `chunk`, an expert's pairs are split
// into runs of at most `chunk` (each run its own entry u, so a tile kernel's
// MMA columns always suffice; such an expert's weights are then read once per
// run).
// `my_id`: ids[threadIdx.x], loaded by the caller ahead of time (when
// threadIdx.x < n).
__device__ __forceinline__ void build_route(const int32_t* __restrict__ ids, int my_id, int n, int E, RouteView r,
                                            int chunk = 1 << 30, int ebase = 0) {
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    // an expert-parallel shard holds experts [ebase, ebase + E)
    const int e = (p == (int)threadIdx.x ? my_id : __ldcg(ids + p)) - ebase;
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
  if (chunk < nv) {  // bit 1: a run start inside an expert (bit 0, read here, stays put)
    for (int k = threadIdx.x; k < nv; k += blockDim.x) {
      if (r.first[k] & 1) continue;
      int j = k;
      while (!(r.first[j] & 1)) j--;
      if ((k - j) % chunk == 0) r.first[k] |= 2;
    }
    __syncthreads();
  }
  for (int k = threadIdx.x; k < nv; k += blockDim.x) {
    if (!r.first[k]) continue;
    int u = 0;
    for (int q = 0; q < k; q++) u += r.first[q] != 0;
    r.uexp[u] = r.ids[r.sorted[k]];
    r.ustart[u] = (int16_t)k;
  }
  if (threadIdx.x == 0) {
    int D = 0;
    for (int q = 0; q < nv; q++) D += r.first[q] != 0;
    r.scalars[0] = D;
    r.ustart[D] = (int16_t)nv;
  }
  __syncthreads();
}

// The same list for at most 32 pairs, built by warp 0 alone (lane p holds
// pair p): stable ranks by ballot and shuffle, run starts by ballot; one CTA
// barrier at the end.
__device__ __forceinline__ void build_route_warp(int my_id, int n, int E, RouteView r, int chunk, int ebase) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int e0 = lane < n ? my_id - ebase : -1;
    const int ev = (lane < n && e0 >= 0 && e0 < E) ? e0 : -1;
    if (lane < n) r.ids[lane] = ev;
    int rank = 0;
    for (int q = 0; q < n; q++) {  // lanes past n hold no pair
      const int eq = __shfl_sync(0xffffffffu, ev, q);
      rank += (eq >= 0) && (eq < ev || (eq == ev && q < lane));
    }
    const int nv = __popc(__ballot_sync(0xffffffffu, ev >= 0));
    if (ev >= 0) r.sorted[rank] = (int16_t)lane;
    __syncwarp();
    // position k of the expert order: its expert, and whether a run starts there
    const int ek = lane < nv ? r.ids[r.sorted[lane]] : -1;
    const int eprev = __shfl_up_sync(0xffffffffu, ek, 1);
    const unsigned bound = __ballot_sync(0xffffffffu, lane < nv && (lane == 0 || eprev != ek));
    const int start = 31 - __clz(bound & (0xffffffffu >> (31 - lane)));  // this expert's first position
    const unsigned runs = __ballot_sync(0xffffffffu, lane < nv && (lane - start) % chunk == 0);
    if ((runs >> lane) & 1u) {
      const int u = __popc(runs & ((1u << lane) - 1u));
      r.uexp[u] = ek;
      r.ustart[u] = (int16_t)lane;
    }
    if (lane == 0) {
      const int D = __popc(runs);
      r.scalars[0] = D;
      r.scalars[1] = nv;
      r.ustart[D] = (int16_t)nv;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------- prep kernel
// Inputs that a routed call reads from page-locked host memory, copied once
// into the workspace by the prep kernel (n = 0, nx = 0: nothing to copy).
struct PrepStage {
  const int32_t* ids;
  const float* p;
  int32_t* ids_out;
  float* p_out;
  int n;  // pairs
  const uint4* xraw;
  uint4* xraw_out;
  int nx;  // 16-byte words of x copied as they are
};

// Resets the status word and records out-of-range expert ids, zeroes the
// stream kernel's tile counters (GEMV) and slot-transposes the activations
// read through L1 (x[t][16w + i + 4j] -> xp[t][16w + 4i + j]); T = 0 skips
// the transposition (x staged in shared memory), npairs = 0 the id check.
// With host-resident inputs it also copies ids, p and (for x staged in
// shared memory) x into the workspace.
__global__ void __launch_bounds__(256) k_prep(const uint16_t* __restrict__ x, int T, int cols,
                                              uint16_t* __restrict__ xp, int32_t* __restrict__ zero,
                                              int nzero, const int32_t* __restrict__ ids, int npairs, int E,
                                              int32_t* __restrict__ status, PrepStage sg) {
  // Launched as a dependent of whatever precedes it (the previous call's last
  // kernel may still be writing this call's x or ids, or reading the
  // workspace written below): nothing is read or written before the wait.
  // Only then may the call's other kernels launch, so they can read the
  // call's inputs as soon as they start.
  griddep_wait();
  griddep_launch();
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int nth = gridDim.x * blockDim.x;
  for (int i = tid; i < nzero; i += nth) zero[i] = 0;
  for (int i = tid; i < sg.n; i += nth) {
    sg.ids_out[i] = sg.ids[i];
    sg.p_out[i] = sg.p[i];
  }
  for (int i = tid; i < sg.nx; i += nth) sg.xraw_out[i] = sg.xraw[i];
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

// ------------------------------------------------------- kernel modes
// An item is 16 rows of one matrix over a slice of `bpi` blocks of the
// reduction width; its MMA columns are the tokens (GEMV) or the (token, slot)
// pairs of one run of a distinct expert (routed modes). Each warp streams
// its items through a ring of kStages stages, one item per stage, so loads
// run up to kStages items ahead of the decode.
//   stream kernel (items spread over every warp of the grid):
//   GEMV:   slices of a tile meet in the workspace; y[t][row] = sum (fp32).
//   FLOOR:  identical loads; the decode is replaced by an XOR of every loaded
//           byte into out[expert][row].
//   tile kernel (a CTA reduces a group of items in shared memory):
//   GATEUP: gate and up slices of a tile; h = bf16(silu(g) * u), slot-transposed.
//   DOWN:   every run's slices of a tile; y = sum_j p_j * (...), bf16.
//   SWITCH: one projection per (token, slot) pair; y[pair][row] (fp32).
enum : int { MODE_GEMV = 0, MODE_GATEUP = 1, MODE_DOWN = 2, MODE_FLOOR = 3, MODE_SWITCH = 4 };

struct UnitArgs {
  WDev w0, w1;
  Values V;
  const int32_t* ids;
  const float* p;
  const uint16_t* act;   // slot-transposed activation rows (read-only path)
  const uint16_t* xraw;  // BSM: the activation rows as given, transposed on the way into shared memory
  int T, topk, expert;
  const int32_t* elist;  // FLOOR: experts to stream
  int nexp;
  float* yf;        // GEMV output [T][rows]; SWITCH output [pairs][rows]
  uint16_t* out16;  // GATEUP: h [pairs][inter]; DOWN: y [T][hidden]
  uint32_t* outx;   // FLOOR: [nexp][rows], zeroed before the launch
  int32_t* cnt;
  float* part;
  int32_t* status;
  int32_t* ready;  // routed decode: per run, gate/up tile groups of h written (gate/up adds, down polls); or null
  int bpi;       // 256-weight blocks per item
  int splits;    // items per tile and matrix (blocks per row / bpi)
  int async_sc;  // scale slices by cp.async (blocks per row a multiple of four)
  int act_rows;  // BSM: activation rows copied into shared memory
  int tpg;       // tile kernel, SWITCH: tiles per group (items per group = splits * tpg)
  int ebase;     // routed modes: first expert id the weights hold (expert-parallel shard)
  int first;     // tile kernel launched as the call's first kernel (no prep kernel before it)
  int wait_in;   // tile kernel: ids, p (and x) are the prep kernel's copies: wait for it before reading them
  int check_ids; // first: record out-of-range ids in the status word
  int expire;    // testing hook: warp 0 of every CTA also waits on a barrier nothing arrives on
  uint64_t wait_ns;  // bound of every wait on a data barrier (global-timer ns)
  FastDiv div_s, div_tiles;
};

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Wait until at most `pending` of this thread's cp.async groups are still in flight.
__device__ __forceinline__ void cp_async_wait_upto(int pending) {
  if (pending <= 0) cp_async_wait_group<0>();
  else if (pending == 1) cp_async_wait_group<1>();
  else if (pending == 2) cp_async_wait_group<2>();
  else cp_async_wait_group<3>();
}
// The mbarrier's current phase also waits for this thread's earlier cp.async copies.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Stage the scale slice of rows [R0, R0 + valid) and blocks [s*bpi, (s+1)*bpi)
// of `w` into `slot`. With `async` (blocks per row a multiple of four and bpi
// 2 or 4, so every row piece is 4-, 8- or 16-byte aligned) the lanes issue
// cp.async copies tracked by `bar`; otherwise they copy with plain loads
// (IQ2_KS sch / sex at window offset 0), zero past the last row, and the call
// ends with __syncwarp.
template <int FMT>
__device__ __forceinline__ void stage_scales(uint8_t* slot, const WDev& w, int64_t R0, int valid, int s, int bpi,
                                             bool async, uint64_t* bar, int lane) {
  const int nbk = w.cols / 256;
  if (async) {
    const int r = lane & 15;
    if (r < valid) {
      const int64_t o = (R0 + r) * nbk + (int64_t)s * bpi;  // first block of the slice in the row's planes
      if (FMT == FMT_KS) {
        if (lane < 16) {
          if (bpi == 4) cp_async16(slot + 16 * r, w.scl + o);
          else cp_async8(slot + 8 * r, w.scl + o);
        } else {
          const int64_t win = o & ~(int64_t)3;
          cp_async4(slot + Slot<FMT>::b_off(bpi) + 4 * r, w.sch + win);
          cp_async4(slot + Slot<FMT>::c_off(bpi) + 4 * r, reinterpret_cast<const uint8_t*>(w.sex) + win);
        }
      } else {
        if (bpi == 4) cp_async16(slot + 32 * r + 16 * (lane >> 4), w.scl + 2 * o + 4 * (lane >> 4));
        else if (lane < 16) cp_async16(slot + 16 * r, w.scl + 2 * o);
        const uint16_t* src = lane < 16 ? reinterpret_cast<const uint16_t*>(w.sex) + o : w.dv + o;
        uint8_t* dst = slot + (lane < 16 ? Slot<FMT>::b_off(bpi) : Slot<FMT>::c_off(bpi)) + 2 * bpi * r;
        if (bpi == 4) cp_async8(dst, src);
        else cp_async4(dst, src);
      }
    }
    if (FMT == FMT_KS) {  // the tile's 16 row scales: two 16-byte copies, or plain loads off the grid
      uint16_t* sdv = reinterpret_cast<uint16_t*>(slot + Slot<FMT>::dv_off(bpi));
      if (valid == kTile && ((reinterpret_cast<uintptr_t>(w.dv + R0) & 15) == 0)) {
        if (lane < 2) cp_async16(sdv + 8 * lane, w.dv + R0 + 8 * lane);
      } else if (lane < kTile) {
        sdv[lane] = lane < valid ? __ldg(w.dv + R0 + lane) : (uint16_t)0;
      }
    }
    cp_async_arrive(bar);
    return;
  }
  if (FMT == FMT_KS) {
    uint32_t* d32 = reinterpret_cast<uint32_t*>(slot);
    for (int i = lane; i < 16 * bpi; i += 32) {
      const int r = i / bpi, b = i - r * bpi;
      d32[i] = r < valid ? __ldg(w.scl + (R0 + r) * nbk + s * bpi + b) : 0u;
    }
    uint8_t* sb = slot + Slot<FMT>::b_off(bpi);
    uint8_t* sc = slot + Slot<FMT>::c_off(bpi);
    for (int i = lane; i < 16 * bpi; i += 32) {
      const int r = i / bpi, b = i - r * bpi;
      const int64_t o = (R0 + r) * nbk + s * bpi + b;
      sb[4 * r + b] = r < valid ? __ldg(w.sch + o) : (uint8_t)0;
      sc[4 * r + b] = r < valid ? __ldg(reinterpret_cast<const uint8_t*>(w.sex) + o) : (uint8_t)0;
    }
    uint16_t* sdv = reinterpret_cast<uint16_t*>(slot + Slot<FMT>::dv_off(bpi));
    if (lane < kTile) sdv[lane] = lane < valid ? __ldg(w.dv + R0 + lane) : (uint16_t)0;
  } else {
    uint32_t* d32 = reinterpret_cast<uint32_t*>(slot);
    for (int i = lane; i < 32 * bpi; i += 32) {
      const int r = i / (2 * bpi), b = i - r * 2 * bpi;
      d32[i] = r < valid ? __ldg(w.scl + (R0 + r) * 2 * nbk + 2 * s * bpi + b) : 0u;
    }
    uint16_t* sb = reinterpret_cast<uint16_t*>(slot + Slot<FMT>::b_off(bpi));
    uint16_t* sc = reinterpret_cast<uint16_t*>(slot + Slot<FMT>::c_off(bpi));
    for (int i = lane; i < 16 * bpi; i += 32) {
      const int r = i / bpi, b = i - r * bpi;
      const int64_t o = (R0 + r) * nbk + s * bpi + b;
      sb[i] = r < valid ? __ldg(reinterpret_cast<const uint16_t*>(w.sex) + o) : (uint16_t)0;
      sc[i] = r < valid ? __ldg(w.dv + o) : (uint16_t)0;
    }
  }
  __syncwarp();
}

// Timeout flag of the floor arm, which has no workspace: cleared by each
// floor call's first kernel, read back by iqk_floor_status.
__device__ int32_t g_floor_status;

template <int MODE, int F0, int F1, int NT, bool BSM>
__global__ void __launch_bounds__(kDecodeWarps * 32, kDecodeMinBlocks(NT)) k_stream(const __grid_constant__ CUtensorMap m0,
                                                                         const __grid_constant__ CUtensorMap m1,
                                                                         const __grid_constant__ UnitArgs A) {
  static_assert(MODE == MODE_GEMV || MODE == MODE_FLOOR, "stream kernel: GEMV or floor");
  extern __shared__ __align__(128) uint8_t smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int K = A.w0.cols;
  const int bpi = A.bpi, S = A.splits;
  const int ldw = 16 * bpi;
  const int stage_words = kTile * ldw;
  const uint32_t slot_b = slot_bytes2<F0, F1>(bpi);
  const uint32_t k65536 = opaque_u32(65536u);
  constexpr int NC = 8 * NT;
  const size_t warp_bytes = (size_t)kStages * (stage_words * 4 + slot_b);
  uint32_t* ring_qs = reinterpret_cast<uint32_t*>(smem + wid * warp_bytes);
  uint8_t* ring_slots = smem + wid * warp_bytes + (size_t)kStages * stage_words * 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecodeWarps * warp_bytes);
  uint64_t* bar = bars + wid * kStages;
  uint64_t* never_bar = bars + kDecodeWarps * kStages;  // nothing arrives on it (expire hook)
  uint2* lut0 = reinterpret_cast<uint2*>(never_bar + 2);
  uint2* lut1 = lut0 + 64;
  uint16_t* act_s = reinterpret_cast<uint16_t*>(lut1 + 64);  // BSM activation rows
  // BSM rows keep each lane's 64-element segment in 80 elements (160 bytes),
  // so the four segments a warp reads at once start in different bank groups
  const int KP = BSM ? K / 64 * 80 : K;  // activation row stride (elements)
  if (threadIdx.x == 0) prefetch_tensormap(&m0);
  if (MODE == MODE_GEMV) build_lut<F0>(lut0, A.V);
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&bar[s], 1);
    if (wid == 0) mbar_init(never_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // This kernel starts only after the call's first kernel has seen the
  // previous work on the stream complete (that kernel waits before it lets
  // its dependents launch), so the call's inputs (x, the expert list) and the
  // weight streams are read right away. The workspace and the outputs, which
  // the first kernel writes, are touched only after the dependency wait.
  // Dependents of this kernel may launch at once: they wait the same way.
  griddep_launch();
  const int D = MODE == MODE_FLOOR ? A.nexp : 1;  // matrices streamed
  const int rows = A.w0.rows;
  const int tiles = (rows + kTile - 1) / kTile;
  const int nitems = D * tiles * S;
  const int W = gridDim.x * kDecodeWarps;
  const int gw = blockIdx.x * kDecodeWarps + wid;
  // item id -> (u, tile, s): the slices of a tile are adjacent
  auto item_of = [&](int id, int& u, int& tile, int& s) {
    const int r = (int)A.div_s.div((uint32_t)id);
    s = id - r * S;
    u = (int)A.div_tiles.div((uint32_t)r);
    tile = r - u * tiles;
  };
  auto expert_of = [&](int u) -> int { return MODE == MODE_FLOOR ? __ldcg(A.elist + u) : A.expert; };
  int issued = 0;  // items this warp has requested
  auto issue = [&](int it) {
    const int id = gw + it * W;
    if (id >= nitems) return;
    issued = it + 1;
    const int st = it % kStages;
    int u, tile, s;
    item_of(id, u, tile, s);
    const int e = expert_of(u);
    const int64_t R0 = (int64_t)e * rows + (int64_t)tile * kTile;
    const int valid = min(kTile, rows - tile * kTile);
    uint8_t* slot = ring_slots + (size_t)st * slot_b;
    if (A.w0.slots) {  // the item's scale-slot image: one bulk copy beside the qs tile
      if (lane == 0) {
        const uint32_t sb = Slot<F0>::bytes(bpi);
        mbar_arrive_expect_tx(&bar[st], (uint32_t)stage_words * 4 + sb);
        tma_load_2d(ring_qs + (size_t)st * stage_words, &m0, s * ldw, (int)R0, &bar[st]);
        bulk_load(slot, A.w0.slots + ((size_t)((int64_t)e * tiles + tile) * S + s) * sb, sb, &bar[st]);
      }
      return;
    }
    stage_scales<F0>(slot, A.w0, R0, valid, s, bpi, A.async_sc, &bar[st], lane);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[st], (uint32_t)stage_words * 4);
      tma_load_2d(ring_qs + (size_t)st * stage_words, &m0, s * ldw, (int)R0, &bar[st]);
    }
  };
  for (int s = 0; s < kStages; s++) issue(s);
  if constexpr (BSM) {  // the call's activation rows, slot-transposed and padded, once per CTA
    const int gpr = K / 16;  // 16-element groups per row
    const int groups = A.act_rows * gpr;
    for (int gi = threadIdx.x; gi < groups; gi += blockDim.x) {
      const int r = gi / gpr, c0 = (gi - r * gpr) * 16;
      uint32_t o[8];
      const uint4* src = reinterpret_cast<const uint4*>(A.xraw + (size_t)gi * 16);
      const uint4 a = ld_cg_u4(src), b = ld_cg_u4(src + 1);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i2 = 0; i2 < 4; i2++) {
        const int wa = i2 >> 1;
        const uint32_t sel = (i2 & 1) ? 0x7632u : 0x5410u;
        o[2 * i2] = prmt(w[wa], w[wa + 2], sel);
        o[2 * i2 + 1] = prmt(w[wa + 4], w[wa + 6], sel);
      }
      uint4* dst = reinterpret_cast<uint4*>(act_s + (size_t)r * KP + (c0 >> 6) * 80 + (c0 & 63));
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    __syncthreads();
  }
  const uint16_t* act_base = BSM ? act_s : A.act;
  constexpr int SEG = BSM ? 80 : 64;    // elements between the segments of lanes t and t + 1
  constexpr int BLKE = BSM ? 320 : 256;  // elements between consecutive 256-weight blocks
  griddep_wait();  // from here on: the workspace (transposed x, counters, partial sums) and the outputs
  int32_t* status = A.status ? A.status : &g_floor_status;
  if (A.expire && wid == 0 && !__all_sync(0xffffffffu, mbar_wait_ns(never_bar, 0, A.wait_ns))) {  // testing hook
    if (lane == 0) atomicOr(status, 2);
    for (int k = 0; k < issued; k++) (void)mbar_wait_ns(&bar[k % kStages], (uint32_t)((k / kStages) & 1), kDrainWaitNs);
    return;
  }

  for (int it = 0;; it++) {
    const int id = gw + it * W;
    if (id >= nitems) break;
    int u, tile, s;
    item_of(id, u, tile, s);
    const uint16_t* bsrc[NT];
#pragma unroll
    for (int n = 0; n < NT; n++) {
      // columns past the last token repeat column 0; their sums are never stored
      const int col = 8 * n + g < A.T ? 8 * n + g : 0;
      bsrc[n] = act_base + (size_t)col * KP + (size_t)s * bpi * BLKE + SEG * t;
      if (!BSM && MODE != MODE_FLOOR) prefetch_l1(bsrc[n]);
    }
    const bool fmt0 = true;
    const bool kfmt = F0 == FMT_K;
    const int st = it % kStages;
    // warp-uniform: a lane that saw the data at the bound must not run on alone
    if (!__all_sync(0xffffffffu, mbar_wait_ns(&bar[st], (uint32_t)((it / kStages) & 1), A.wait_ns))) {
      if (lane == 0) atomicOr(status, 2);
      // let this warp's copies still in flight land before the CTA exits
      for (int k = it; k < issued; k++)
        (void)mbar_wait_ns(&bar[k % kStages], (uint32_t)((k / kStages) & 1), kDrainWaitNs);
      return;
    }
    const uint32_t* sq = ring_qs + (size_t)st * stage_words;
    const uint8_t* slot = ring_slots + (size_t)st * slot_b;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) acc[n][q] = 0.f;
    uint32_t xg = 0, xh = 0;  // FLOOR checksums of rows g and g + 8
    if (MODE == MODE_FLOOR) {
      for (int b = 0; b < bpi; b++) {
        const uint4 a4 = *reinterpret_cast<const uint4*>(sq + g * ldw + b * 16 + 4 * t);
        const uint4 b4 = *reinterpret_cast<const uint4*>(sq + (g + 8) * ldw + b * 16 + 4 * t);
        xg ^= a4.x ^ a4.y ^ a4.z ^ a4.w;
        xh ^= b4.x ^ b4.y ^ b4.z ^ b4.w;
      }
      // the slice's scale bytes; byte j of a row's plane lands in byte j & 3
      const bool ks = F0 == FMT_KS;
      const uint32_t* s32 = reinterpret_cast<const uint32_t*>(slot);
      const int nw = ks ? bpi : 2 * bpi;  // scl words per row (slices start on word boundaries)
      for (int i = t; i < nw; i += 4) {
        xg ^= s32[g * nw + i];
        xh ^= s32[(g + 8) * nw + i];
      }
      if (ks) {
        const uint8_t* sb = slot + Slot<FMT_KS>::b_off(bpi);
        const uint8_t* sc = slot + Slot<FMT_KS>::c_off(bpi);
        const int o = (A.async_sc && !A.w0.slots) ? (s * bpi) & 3 : 0;  // window offset (0 in an image)
        for (int i = t; i < bpi; i += 4) {
          const int sh = 8 * ((s * bpi + i) & 3);
          xg ^= ((uint32_t)sb[g * 4 + o + i] ^ (uint32_t)sc[g * 4 + o + i]) << sh;
          xh ^= ((uint32_t)sb[(g + 8) * 4 + o + i] ^ (uint32_t)sc[(g + 8) * 4 + o + i]) << sh;
        }
        if (s == 0 && t == 0) {  // the row scale belongs to the first slice (zero past the last row)
          const uint16_t* sdv = reinterpret_cast<const uint16_t*>(slot + Slot<FMT_KS>::dv_off(bpi));
          xg ^= sdv[g];
          xh ^= sdv[g + 8];
        }
      } else {
        const uint16_t* sb = reinterpret_cast<const uint16_t*>(slot + Slot<FMT_K>::b_off(bpi));
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(slot + Slot<FMT_K>::c_off(bpi));
        for (int i = t; i < bpi; i += 4) {
          const int sh = 16 * ((s * bpi + i) & 1);
          xg ^= ((uint32_t)sb[g * bpi + i] ^ (uint32_t)sc[g * bpi + i]) << sh;
          xh ^= ((uint32_t)sb[(g + 8) * bpi + i] ^ (uint32_t)sc[(g + 8) * bpi + i]) << sh;
        }
      }
    } else {
      const int o = (A.async_sc && !A.w0.slots) ? (s * bpi) & 3 : 0;  // window offset (0 in an image)
      // IQ2_KS row scales of rows g and g + 8, applied after the slice's MMAs
      const float dg = kfmt ? 0.f : d_smem_ks(slot, bpi, g), dh = kfmt ? 0.f : d_smem_ks(slot, bpi, g + 8);
      // unrolled over the item's blocks where registers allow (one or two column groups)
      if (NT <= 2 && bpi == 4)
        item_mma<F0, F1, NT, BSM, 4>(sq, slot, bpi, o, ldw, bsrc, fmt0, kfmt, lut0, lut1, dg, dh, g, t, k65536, acc);
      else if (NT <= 2 && bpi == 2)
        item_mma<F0, F1, NT, BSM, 2>(sq, slot, bpi, o, ldw, bsrc, fmt0, kfmt, lut0, lut1, dg, dh, g, t, k65536, acc);
      else
        item_mma<F0, F1, NT, BSM>(sq, slot, bpi, o, ldw, bsrc, fmt0, kfmt, lut0, lut1, dg, dh, g, t, k65536, acc);
    }
    __syncwarp();
    issue(it + kStages);  // refill the stage just consumed

    const int rg = tile * kTile + g, rh = rg + 8;
    if (MODE == MODE_FLOOR) {
      xg ^= __shfl_xor_sync(0xffffffffu, xg, 1);
      xg ^= __shfl_xor_sync(0xffffffffu, xg, 2);
      xh ^= __shfl_xor_sync(0xffffffffu, xh, 1);
      xh ^= __shfl_xor_sync(0xffffffffu, xh, 2);
      if (t == 0) {
        if (rg < rows) atomicXor(A.outx + (size_t)u * rows + rg, xg);
        if (rh < rows) atomicXor(A.outx + (size_t)u * rows + rh, xh);
      }
      continue;
    }

    if (MODE == MODE_GEMV) {
      if (S == 1) {
#pragma unroll
        for (int n = 0; n < NT; n++)
#pragma unroll
          for (int q = 0; q < 4; q++) {
            const int col = 8 * n + 2 * t + (q & 1);
            const int row = tile * kTile + g + 8 * (q >> 1);
            if (col < A.T && row < rows) A.yf[(size_t)col * rows + row] = acc[n][q];
          }
        continue;
      }
      float* slotp = A.part + ((size_t)tile * S + s) * NC * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) slotp[(8 * n + 2 * t + (q & 1)) * kTile + g + 8 * (q >> 1)] = acc[n][q];
      __syncwarp();
      int prev = 0;
      if (lane == 0) {
        __threadfence();
        prev = atomicAdd(A.cnt + tile, 1);
      }
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != S - 1) continue;
      __threadfence();
      const float* base = A.part + (size_t)tile * S * NC * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const int col = 8 * n + 2 * t + (q & 1);
          const int r = g + 8 * (q >> 1);
          const int row = tile * kTile + r;
          if (col >= A.T || row >= rows) continue;
          float sum = 0.f;
          for (int ss = 0; ss < S; ss++) sum += __ldcg(base + ((size_t)ss * NC + col) * kTile + r);
          A.yf[(size_t)col * rows + row] = sum;
        }
    }
  }
}

// ------------------------------------------------------------- tile kernel
// Gate/up and down with the slices of an output tile reduced inside one CTA
// (one or two MMA column groups). A CTA takes tile groups in turn, group
// blockIdx.x + r * gridDim.x in round r:
//   GATEUP: group = (distinct expert u, 16-row tile of the intermediate
//           dimension); its items are the gate and up slices, 2 * S of them;
//   DOWN:   group = 16-row tile of the hidden dimension; its items are the
//           (distinct expert, slice) pairs, D * S of them.
// Warp w takes items w, w + kDecodeWarps, ... of each group and adds them into
// its own shared-memory slot; after a CTA barrier the threads sum the slots in
// warp order (the same order every call) and write h = bf16(silu(g) * u) or
// y = bf16(sum over slots of p * down). No device-scope counters are needed.
template <int MODE, int F0, int F1, int NT, bool BSM>
__global__ void __launch_bounds__(kDecodeWarps * 32, kDecodeMinBlocks(NT)) k_tiles(const __grid_constant__ CUtensorMap m0,
                                                                             const __grid_constant__ CUtensorMap m1,
                                                                             const __grid_constant__ UnitArgs A) {
  static_assert(MODE == MODE_GATEUP || MODE == MODE_DOWN || MODE == MODE_SWITCH, "tile kernel: gate/up, down, switch");
  extern __shared__ __align__(128) uint8_t smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int K = A.w0.cols;
  const int bpi = A.bpi, S = A.splits;
  const int ldw = 16 * bpi;
  const int stage_words = kTile * ldw;
  const uint32_t slot_b = slot_bytes2<F0, F1>(bpi);
  const uint32_t k65536 = opaque_u32(65536u);
  constexpr int NC = 8 * NT;
  const int npairs = A.T * A.topk;
  const size_t warp_bytes = (size_t)kStages * (stage_words * 4 + slot_b);
  uint32_t* ring_qs = reinterpret_cast<uint32_t*>(smem + wid * warp_bytes);
  uint8_t* ring_slots = smem + wid * warp_bytes + (size_t)kStages * stage_words * 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecodeWarps * warp_bytes);
  uint64_t* bar = bars + wid * kStages;
  uint64_t* never_bar = bars + kDecodeWarps * kStages;  // nothing arrives on it (expire hook)
  uint2* lut0 = reinterpret_cast<uint2*>(never_bar + 2);
  uint2* lut1 = lut0 + 64;
  const int KP = BSM ? K / 64 * 80 : K;  // activation row stride (elements), see k_stream
  uint16_t* act_s = reinterpret_cast<uint16_t*>(lut1 + 64);
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(act_s) + (BSM ? (size_t)A.act_rows * KP * 2 : 0));
  // floats per warp slot: (mat, column, row) gate/up; (column, row) switch; (token, row) down
  const int slot_f = MODE == MODE_GATEUP ? 2 * NC * kTile : MODE == MODE_SWITCH ? NC * kTile : A.T * kTile;
  uint8_t* route_p = reinterpret_cast<uint8_t*>(red + (size_t)kDecodeWarps * slot_f);
  // This kernel starts only after the call's first kernel has seen the
  // previous work on the stream complete (that kernel waits before it lets
  // its dependents launch), so the call's inputs (x, ids, p) and the weight
  // streams are read right away: the routing is built and the first weight
  // tiles are requested while the preceding kernel of this call finishes.
  // What a preceding kernel of the call writes (the status word, transposed
  // x, h) and the outputs are touched only after the dependency wait.
  // Dependents of this kernel may launch at once: they wait the same way.
  // As the call's first kernel (A.first) it waits for everything before it
  // first, like the prep kernel it replaces, and only then lets the call's
  // other kernels launch.
  if (threadIdx.x == 0) {
    prefetch_tensormap(&m0);
    if (MODE == MODE_GATEUP) prefetch_tensormap(&m1);
  }
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&bar[s], 1);
    if (wid == 0) mbar_init(never_bar, 1);
    fence_mbar_init();
  }
  // Routed decode with per-run readiness (A.ready): the gate/up kernel adds
  // one to a run's counter after each of the run's tile groups of h, and the
  // down kernel, which has no dependency wait before its items, copies a
  // run's h once the run's counter is complete; it waits for the gate/up
  // kernel only before it writes y. The prep kernel zeroes the counters, and
  // the gate/up kernel lets the down kernel launch only after its own
  // dependency wait has seen the prep kernel complete, so the down kernel
  // never reads a counter of an earlier call.
  const bool publish = MODE == MODE_GATEUP && A.ready != nullptr;
  const bool hready = MODE == MODE_DOWN && BSM && A.ready != nullptr;
  if (A.first || A.wait_in) griddep_wait();
  if (!publish) griddep_launch();
  // the call's inputs first (ids, routing weights, x), then the tables while they arrive
  // (switch mode without an ids array: every pair is on expert A.expert, a
  // single-matrix GEMV of at most 4 tokens, whose routing the warp builds)
  const int my_id = (int)threadIdx.x >= npairs ? 0
                    : (MODE == MODE_SWITCH && !A.ids) ? A.expert
                                                      : __ldcg(A.ids + threadIdx.x);
  const float my_p = (MODE == MODE_DOWN && (int)threadIdx.x < npairs) ? __ldcg(A.p + threadIdx.x) : 0.f;
  // gate/up and switch: request the first activation groups ahead of the weight stream
  uint4 pre0 = make_uint4(0u, 0u, 0u, 0u), pre1 = pre0, pre2 = pre0, pre3 = pre0;
  const int act_groups = BSM ? A.act_rows * (K / 16) : 0;
  if (BSM && MODE != MODE_DOWN) {
    const int g0 = threadIdx.x, g1 = threadIdx.x + blockDim.x;
    if (g0 < act_groups) {
      pre0 = ld_cg_u4(A.xraw + (size_t)g0 * 16);
      pre1 = ld_cg_u4(A.xraw + (size_t)g0 * 16 + 8);
    }
    if (g1 < act_groups) {
      pre2 = ld_cg_u4(A.xraw + (size_t)g1 * 16);
      pre3 = ld_cg_u4(A.xraw + (size_t)g1 * 16 + 8);
    }
  }
  build_lut<F0>(lut0, A.V);
  if (MODE == MODE_GATEUP) build_lut<F1>(lut1, A.V);
  const RouteView rt = carve_route(route_p, npairs);
  if (MODE == MODE_DOWN)  // the routing weights, read once per pair and item below
    for (int i = threadIdx.x; i < npairs; i += blockDim.x) rt.pw[i] = i == (int)threadIdx.x ? my_p : __ldcg(A.p + i);
  // ends with __syncthreads; runs of <= NC pairs
  if (npairs <= 32) build_route_warp(my_id, npairs, A.w0.experts, rt, NC, A.ebase);
  else build_route(A.ids, my_id, npairs, A.w0.experts, rt, NC, A.ebase);
  const int D = rt.scalars[0];
  const int rows = A.w0.rows;
  const int tiles = (rows + kTile - 1) / kTile;
  // SWITCH: a group is `tpg` consecutive tiles of one expert (the last run
  // may extend past the matrix: those items load its last tile and are dropped)
  const int tpg = MODE == MODE_SWITCH ? A.tpg : 1;
  const int ntg = (tiles + tpg - 1) / tpg;  // groups per expert (SWITCH)
  const int n_it = MODE == MODE_GATEUP ? 2 * S : MODE == MODE_SWITCH ? S * tpg : D * S;  // items per group
  const int ngroups = MODE == MODE_GATEUP ? D * tiles : MODE == MODE_SWITCH ? D * ntg : tiles;
  const int rounds = (int)blockIdx.x < ngroups ? (ngroups - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int cnt_w = wid < n_it ? (n_it - 1 - wid) / kDecodeWarps + 1 : 0;  // this warp's items per group
  const int nq = rounds * cnt_w;
  // q-th item of this warp -> (u, mat, tile, s)
  auto item_at = [&](int q, int& u, int& mat, int& tile, int& s) {
    const int r = q / cnt_w;
    const int j = wid + (q - r * cnt_w) * kDecodeWarps;
    const int tg = (int)blockIdx.x + r * (int)gridDim.x;
    const int js = (int)A.div_s.div((uint32_t)j);
    s = j - js * S;
    if (MODE == MODE_GATEUP) {
      mat = js;
      u = (int)A.div_tiles.div((uint32_t)tg);
      tile = tg - u * tiles;
    } else if (MODE == MODE_SWITCH) {
      mat = 0;
      u = (int)A.div_tiles.div((uint32_t)tg);  // div_tiles divides by ntg here
      tile = min((tg - u * ntg) * tpg + js, tiles - 1);
    } else {
      mat = 0;
      u = js;
      tile = tg;
    }
  };
  int issued = 0;
  auto issue = [&](int q) {
    if (q >= nq) return;
    const int st = q % kStages;
    int u, mat, tile, s;
    item_at(q, u, mat, tile, s);
    const int e = rt.uexp[u];
    const int64_t R0 = (int64_t)e * rows + (int64_t)tile * kTile;
    const int valid = min(kTile, rows - tile * kTile);
    uint8_t* slot = ring_slots + (size_t)st * slot_b;
    issued = q + 1;
    const uint8_t* images = mat ? A.w1.slots : A.w0.slots;
    if (images) {  // the item's scale-slot image: one bulk copy beside the qs tile
      if (lane == 0) {
        const uint32_t sb = mat ? Slot<F1>::bytes(bpi) : Slot<F0>::bytes(bpi);
        mbar_arrive_expect_tx(&bar[st], (uint32_t)stage_words * 4 + sb);
        tma_load_2d(ring_qs + (size_t)st * stage_words, mat ? &m1 : &m0, s * ldw, (int)R0, &bar[st]);
        bulk_load(slot, images + ((size_t)((int64_t)e * tiles + tile) * S + s) * sb, sb, &bar[st]);
      }
      return;
    }
    if (mat == 0) stage_scales<F0>(slot, A.w0, R0, valid, s, bpi, A.async_sc, &bar[st], lane);
    else stage_scales<F1>(slot, A.w1, R0, valid, s, bpi, A.async_sc, &bar[st], lane);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[st], (uint32_t)stage_words * 4);
      tma_load_2d(ring_qs + (size_t)st * stage_words, mat ? &m1 : &m0, s * ldw, (int)R0, &bar[st]);
    }
  };
  for (int q = 0; q < kStages; q++) issue(q);
  // from here on: what the call's preceding kernels wrote, and the outputs
  // (the down kernel with per-run readiness: h through the run counters).
  // A gate/up kernel that publishes runs and stages x itself needs nothing
  // the prep kernel writes before its first counter add: it waits there.
  const bool late_wait = publish && BSM;
  if (!A.first && !hready && !late_wait) griddep_wait();
  if (publish && !late_wait) griddep_launch();
  // The first kernel resets the call's status word (and records ids outside
  // [0, E)). Every other write to it is a timeout bit, set at least one wait
  // bound after this kernel's CTAs have passed their dependency wait, so
  // after this reset.
  if (A.first && blockIdx.x == 0 && threadIdx.x == 0)
    *reinterpret_cast<volatile int32_t*>(A.status) = (A.check_ids && rt.scalars[1] < npairs) ? 1 : 0;
  if constexpr (BSM) {  // activation rows, slot-transposed and padded, once per CTA
    const int gpr = K / 16;
    for (int k = 0; !hready; k++) {
      const int gi = threadIdx.x + k * blockDim.x;
      if (gi >= act_groups) break;
      const int r = gi / gpr, c0 = (gi - r * gpr) * 16;
      uint32_t o[8];
      if (MODE == MODE_DOWN) {
        const uint4* src = reinterpret_cast<const uint4*>(A.act + (size_t)gi * 16);
        const uint4 a = ld_u4(src), b = ld_u4(src + 1);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(A.xraw + (size_t)gi * 16);
        const uint4 a = k == 0 ? pre0 : k == 1 ? pre2 : ld_cg_u4(src);
        const uint4 b = k == 0 ? pre1 : k == 1 ? pre3 : ld_cg_u4(src + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i2 = 0; i2 < 4; i2++) {
          const int wa = i2 >> 1;
          const uint32_t sel = (i2 & 1) ? 0x7632u : 0x5410u;
          o[2 * i2] = prmt(w[wa], w[wa + 2], sel);
          o[2 * i2 + 1] = prmt(w[wa + 4], w[wa + 6], sel);
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(act_s + (size_t)r * KP + (c0 >> 6) * 80 + (c0 & 63));
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    __syncthreads();
  }
  if (MODE == MODE_SWITCH && rt.scalars[1] < npairs) {  // out-of-range ids: zero rows
    for (int pr = 0; pr < npairs; pr++) {
      if (rt.ids[pr] >= 0) continue;
      for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += gridDim.x * blockDim.x)
        A.yf[(size_t)pr * rows + i] = 0.f;
    }
  }
  if (MODE == MODE_DOWN && D == 0) {  // no pair on these experts: the block output is zero
    if (hready) griddep_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < A.T * rows; i += gridDim.x * blockDim.x) {
      if (A.yf) A.yf[i] = 0.f;
      else A.out16[i] = 0;
    }
    return;
  }
  const uint16_t* act_base = BSM ? act_s : A.act;
  constexpr int SEG = BSM ? 80 : 64;
  constexpr int BLKE = BSM ? 320 : 256;
  float* my = red + (size_t)wid * slot_f;
  bool failed = false;
  if (A.expire && wid == 0 && !mbar_wait_ns(never_bar, 0, A.wait_ns)) {  // testing hook: this wait runs out
    failed = true;  // keep taking part in the CTA barriers; stop loading
    if (lane == 0) atomicOr(A.status, 2);
  }
  // Per-run readiness (down kernel): in the first round each warp copies,
  // for each of its items (run u, slice s), that slice of the run's h rows
  // into shared memory itself (cp.async through L2, one commit group per
  // item, in item order) once the run's counter is complete; no other warp
  // touches that slice, and later rounds reuse it. Lane j polls the counter
  // of the warp's j-th pending item: with an acquire load where the warp
  // waits for an item, and with a relaxed load issued before the current
  // item's arithmetic and read after it (look-ahead), in which case the
  // lanes that saw a complete counter read it again with acquire before any
  // copy. A warp barrier passes the acquiring lanes' ordering to the others.
  const int h_target = (K + kTile - 1) / kTile;  // gate/up tile groups per run
  int h_issued = 0;
  auto stage_h = [&](int k) {
    int u, mat, tile, s;
    item_at(k, u, mat, tile, s);
    const int p0 = rt.ustart[u], ncols = rt.ustart[u + 1] - p0;
    const int gps = bpi * 16;  // 16-element groups per slice row
    for (int i = lane; i < ncols * gps; i += 32) {
      const int c = i / gps;
      const int c0 = (s * gps + (i - c * gps)) * 16;
      const int pair = rt.sorted[p0 + c];
      uint16_t* dst = act_s + (size_t)pair * KP + (c0 >> 6) * 80 + (c0 & 63);
      const uint16_t* src = A.act + (size_t)pair * K + c0;
      cp_async16(dst, src);
      cp_async16(dst + 8, src + 8);
    }
    cp_async_commit();
    h_issued = k + 1;
  };
  // the counter of pending item h_issued + lane (-1: none)
  auto poll = [&](bool acquire) -> int32_t {
    const int j = h_issued + lane;
    if (j >= cnt_w) return -1;
    int u, mat, tile, s;
    item_at(j, u, mat, tile, s);
    return acquire ? ld_acquire_s32(A.ready + u) : ld_relaxed_s32(A.ready + u);
  };
  // stage the pending items whose runs are complete, in order, from polled values
  auto stage_ready = [&](int32_t seen, bool acquired) {
    const unsigned m = __ballot_sync(0xffffffffu, seen >= h_target);
    const int n = ~m ? __ffs(~m) - 1 : 32;  // consecutive complete runs from h_issued
    if (n == 0) return;
    if (!acquired && lane < n) {  // counters only grow: this read is complete too, now with acquire
      int u, mat, tile, s;
      item_at(h_issued + lane, u, mat, tile, s);
      (void)ld_acquire_s32(A.ready + u);
    }
    __syncwarp();
    const int stop = min(h_issued + n, cnt_w);
    while (h_issued < stop) stage_h(h_issued);
  };
  int consumed = 0;
  int q = 0;
  for (int r = 0; r < rounds; r++) {
    for (int i = lane; i < slot_f; i += 32) my[i] = 0.f;
    __syncwarp();
    for (int k = 0; k < cnt_w; k++, q++) {
      int u, mat, tile, s;
      item_at(q, u, mat, tile, s);
      const int p0 = rt.ustart[u];
      const int ncols = rt.ustart[u + 1] - p0;
      const uint16_t* bsrc[NT];
#pragma unroll
      for (int n = 0; n < NT; n++) {
        // columns past the last pair repeat column 0; their sums are never used
        const int col = 8 * n + g < ncols ? 8 * n + g : 0;
        const int pair = rt.sorted[p0 + col];
        const int arow = MODE == MODE_DOWN ? pair : pair / A.topk;
        bsrc[n] = act_base + (size_t)arow * KP + (size_t)s * bpi * BLKE + SEG * t;
        if (!BSM) prefetch_l1(bsrc[n]);
      }
      const bool fmt0 = (MODE != MODE_GATEUP) || mat == 0;
      const bool kfmt = fmt0 ? (F0 == FMT_K) : (F1 == FMT_K);
      float acc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int qq = 0; qq < 4; qq++) acc[n][qq] = 0.f;
      int32_t ahead = -1;  // the next pending item's counter, polled during this item
      if (hready && r == 0) {
        failed = __any_sync(0xffffffffu, failed);  // the polls below take the whole warp
        if (!failed && h_issued <= k) {  // this item's slice is not staged: wait (bounded) for its run
          const uint64_t t0 = globaltimer_ns();
          for (;;) {
            stage_ready(poll(true), true);
            if (h_issued > k) break;
            if (__any_sync(0xffffffffu, globaltimer_ns() - t0 >= A.wait_ns)) {
              failed = true;
              if (lane == 0) atomicOr(A.status, 2);
              break;
            }
            __nanosleep(64);
          }
        }
        cp_async_wait_upto(h_issued - (k + 1));  // this item's group (and those before it) have landed
        __syncwarp();
        if (!failed && h_issued < cnt_w) ahead = poll(false);
      }
      const bool polled = hready && r == 0 && !failed && h_issued < cnt_w;
      const int st = q % kStages;
      if (!failed && !mbar_wait_ns(&bar[st], (uint32_t)((q / kStages) & 1), A.wait_ns)) {
        failed = true;  // keep taking part in the CTA barriers; stop loading
        if (lane == 0) atomicOr(A.status, 2);
      }
      if (!failed) {
        consumed = q + 1;
        const uint32_t* sq = ring_qs + (size_t)st * stage_words;
        const uint8_t* slot = ring_slots + (size_t)st * slot_b;
        const int o = (A.async_sc && !(mat ? A.w1.slots : A.w0.slots)) ? (s * bpi) & 3 : 0;  // 0 in an image
        const float dg = kfmt ? 0.f : d_smem_ks(slot, bpi, g), dh = kfmt ? 0.f : d_smem_ks(slot, bpi, g + 8);
        if (bpi == 4)
          item_mma<F0, F1, NT, BSM, 4>(sq, slot, bpi, o, ldw, bsrc, fmt0, kfmt, lut0, lut1, dg, dh, g, t, k65536, acc);
        else if (bpi == 2)
          item_mma<F0, F1, NT, BSM, 2>(sq, slot, bpi, o, ldw, bsrc, fmt0, kfmt, lut0, lut1, dg, dh, g, t, k65536, acc);
        else
          item_mma<F0, F1, NT, BSM>(sq, slot, bpi, o, ldw, bsrc, fmt0, kfmt, lut0, lut1, dg, dh, g, t, k65536, acc);
        __syncwarp();
        issue(q + kStages);  // refill the stage just consumed
      }
      if (polled) stage_ready(ahead, false);  // later items whose runs completed meanwhile
      // add into this warp's slot: (mat, column, row) for gate/up, (column, row)
      // for switch (a warp's items in a group share one tile), (token, row) for down
      if (MODE != MODE_DOWN) {
#pragma unroll
        for (int n = 0; n < NT; n++)
#pragma unroll
          for (int qq = 0; qq < 4; qq++)
            my[(mat * NC + 8 * n + 2 * t + (qq & 1)) * kTile + g + 8 * (qq >> 1)] += acc[n][qq];
      } else {
        // one column (pair) at a time: a token may list one expert twice
        for (int c = 0; c < ncols; c++) {
#pragma unroll
          for (int n = 0; n < NT; n++)
#pragma unroll
            for (int qq = 0; qq < 4; qq++) {
              if (8 * n + 2 * t + (qq & 1) != c) continue;
              const int pair = rt.sorted[p0 + c];
              my[(pair / A.topk) * kTile + g + 8 * (qq >> 1)] += rt.pw[pair] * acc[n][qq];
            }
          __syncwarp();
        }
      }
      __syncwarp();
    }
    __syncthreads();  // every warp's slot of this group is complete
    if (hready) griddep_wait();  // y only after the gate/up kernel has completed
    const int tg = (int)blockIdx.x + r * (int)gridDim.x;
    if (MODE == MODE_GATEUP) {
      const int u = (int)A.div_tiles.div((uint32_t)tg);
      const int tile = tg - u * tiles;
      const int p0 = rt.ustart[u];
      const int ncols = min(rt.ustart[u + 1] - p0, NC);  // runs never exceed NC; the bound guards the slot reads
      for (int o = threadIdx.x; o < ncols * kTile; o += blockDim.x) {
        const int col = o / kTile, row = o - col * kTile;
        const int f = tile * kTile + row;
        if (f >= rows) continue;
        float gv = 0.f, uv = 0.f;
        for (int w = 0; w < kDecodeWarps; w++) {
          gv += red[(size_t)w * slot_f + col * kTile + row];
          uv += red[(size_t)w * slot_f + (NC + col) * kTile + row];
        }
        const float h = silu_f32(gv) * uv;
        A.out16[(size_t)rt.sorted[p0 + col] * rows + perm16(f)] = f32_to_bf16_bits(h);
      }
    } else if (MODE == MODE_SWITCH) {
      // y[pair][row] = sum of the tile's slices; with several tiles per group
      // warp w holds slice w % S of tile w / S (one item each)
      const int u = (int)A.div_tiles.div((uint32_t)tg);
      const int t0 = (tg - u * ntg) * tpg;
      const int p0 = rt.ustart[u];
      const int ncols = min(rt.ustart[u + 1] - p0, NC);
      const int per = ncols * kTile;
      for (int o = threadIdx.x; o < tpg * per; o += blockDim.x) {
        const int sub = o / per, rem = o - sub * per;
        const int col = rem / kTile, row = rem - col * kTile;
        const int f = (t0 + sub) * kTile + row;
        if (t0 + sub >= tiles || f >= rows) continue;
        const int w0 = tpg > 1 ? sub * S : 0, w1 = tpg > 1 ? w0 + S : kDecodeWarps;
        float v = 0.f;
        for (int w = w0; w < w1; w++) v += red[(size_t)w * slot_f + col * kTile + row];
        A.yf[(size_t)rt.sorted[p0 + col] * rows + f] = v;
      }
    } else {
      for (int o = threadIdx.x; o < A.T * kTile; o += blockDim.x) {
        const int tok = o / kTile, row = o - tok * kTile;
        const int f = tg * kTile + row;
        if (f >= rows) continue;
        float y = 0.f;
        for (int w = 0; w < kDecodeWarps; w++) y += red[(size_t)w * slot_f + tok * kTile + row];
        if (A.yf) A.yf[(size_t)tok * rows + f] = y;  // an expert-parallel partial, summed across ranks
        else A.out16[(size_t)tok * rows + f] = f32_to_bf16_bits(y);
      }
    }
    __syncthreads();  // slots free for the next group
    if (late_wait && r == 0) {  // the prep kernel has zeroed the run counters: the down kernel may start
      griddep_wait();
      griddep_launch();
    }
    if (publish && threadIdx.x == 0) {  // one more tile group of this run is in h (the barrier above
      // orders every thread's h stores before this release)
      asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(A.ready + (int)A.div_tiles.div((uint32_t)tg))
                   : "memory");
    }
  }
  // let copies still in flight land before the CTA exits (only after a timeout)
  for (int qd = consumed; qd < issued; qd++) (void)mbar_wait_ns(&bar[qd % kStages], (uint32_t)((qd / kStages) & 1), kDrainWaitNs);
  if (hready) cp_async_wait_group<0>();
}

// ------------------------------------------------------ scale-slot images
// For every (expert, 16-row tile, reduction slice of bpi blocks) of a weight
// tensor, the bytes a decode item stages into its shared-memory slot, in the
// slot layout above with window offset 0 and zeros past the last row (and in
// the IQ2_KS sch / sex row windows past the slice's bpi bytes). Image
// (e, tile, s) sits at ((e * tiles + tile) * S + s) * Slot<FMT>::bytes(bpi).
// The bytes are the planes' own; only their order changes, as the page's
// build-time stream relayout does, so an item fetches its scales with one
// bulk copy. One thread per (image, row).
template <int FMT>
__global__ void __launch_bounds__(256) k_pack_slots(WDev w, int bpi, uint8_t* __restrict__ out) {
  const int tiles = (w.rows + kTile - 1) / kTile;
  const int nbk = w.cols / 256;
  const int S = nbk / bpi;
  const uint32_t SB = Slot<FMT>::bytes(bpi);
  const int64_t n = (int64_t)w.experts * tiles * S * kTile;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i % kTile);
    const int64_t img = i / kTile;
    const int s = (int)(img % S);
    const int64_t et = img / S;  // e * tiles + tile
    const int tile = (int)(et % tiles);
    const int64_t e = et / tiles;
    const int row = tile * kTile + r;
    const bool valid = row < w.rows;
    const int64_t R = e * w.rows + row;
    uint8_t* slot = out + img * SB;
    if (FMT == FMT_KS) {
      uint32_t* d32 = reinterpret_cast<uint32_t*>(slot);
      for (int b = 0; b < bpi; b++) d32[r * bpi + b] = valid ? __ldg(w.scl + R * nbk + s * bpi + b) : 0u;
      uint8_t* sb = slot + Slot<FMT>::b_off(bpi);
      uint8_t* sc = slot + Slot<FMT>::c_off(bpi);
      for (int b = 0; b < 4; b++) {
        const bool in = valid && b < bpi;
        sb[4 * r + b] = in ? __ldg(w.sch + R * nbk + s * bpi + b) : (uint8_t)0;
        sc[4 * r + b] = in ? __ldg(reinterpret_cast<const uint8_t*>(w.sex) + R * nbk + s * bpi + b) : (uint8_t)0;
      }
      reinterpret_cast<uint16_t*>(slot + Slot<FMT>::dv_off(bpi))[r] = valid ? __ldg(w.dv + R) : (uint16_t)0;
    } else {
      uint32_t* d32 = reinterpret_cast<uint32_t*>(slot);
      for (int b = 0; b < 2 * bpi; b++) d32[r * 2 * bpi + b] = valid ? __ldg(w.scl + R * 2 * nbk + 2 * s * bpi + b) : 0u;
      uint16_t* sb = reinterpret_cast<uint16_t*>(slot + Slot<FMT>::b_off(bpi));
      uint16_t* sc = reinterpret_cast<uint16_t*>(slot + Slot<FMT>::c_off(bpi));
      for (int b = 0; b < bpi; b++) {
        sb[r * bpi + b] = valid ? __ldg(reinterpret_cast<const uint16_t*>(w.sex) + R * nbk + s * bpi + b) : (uint16_t)0;
        sc[r * bpi + b] = valid ? __ldg(w.dv + R * nbk + s * bpi + b) : (uint16_t)0;
      }
    }
  }
}

// ================================================================== host

// Bound of the data-barrier waits and the expire hook, copied into every
// decode-side launch (iqk_set_wait_limit_ns).
static std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
static std::atomic<int> g_expire{0};

void set_wait_limit(uint64_t ns, int expire) {
  g_wait_ns.store(ns ? ns : kDefaultWaitNs);
  g_expire.store(expire ? 1 : 0);
}

int read_floor_status(cudaStream_t st, int32_t* out) {
  if (cudaStreamSynchronize(st) != cudaSuccess) return -4;
  return cudaMemcpyFromSymbol(out, g_floor_status, sizeof(int32_t)) == cudaSuccess ? 0 : -4;
}

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

// Activation rows staged in shared memory (padded by 5/4) when they fit this budget.
constexpr size_t kActSmemMax = 40 * 1024;

template <int F0, int F1>
static size_t stream_smem(int cols, int act_rows) {
  const int bpi = item_blocks(cols);
  const size_t warp = (size_t)kStages * ((size_t)kTile * bpi * 16 * 4 + slot_bytes2<F0, F1>(bpi));
  return kDecodeWarps * warp + (size_t)kDecodeWarps * kStages * 8 + 16 + 2 * 64 * 8 +
         (size_t)act_rows * (cols / 64 * 80) * 2;
}

template <int MODE, int F0, int F1, int NT>
static size_t tiles_smem(int cols, int T, int npairs, int act_rows) {
  const int bpi = item_blocks(cols);
  const size_t warp = (size_t)kStages * ((size_t)kTile * bpi * 16 * 4 + slot_bytes2<F0, F1>(bpi));
  const size_t red =
      (size_t)kDecodeWarps * (MODE == MODE_GATEUP ? 2 * 8 * NT * kTile : MODE == MODE_SWITCH ? 8 * NT * kTile : T * kTile) * 4;
  return kDecodeWarps * warp + (size_t)kDecodeWarps * kStages * 8 + 16 + 2 * 64 * 8 + (size_t)act_rows * (cols / 64 * 80) * 2 +
         red + route_smem_bytes(npairs);
}

static int nt_for(int cols_needed) { return cols_needed <= 8 ? 1 : cols_needed <= 16 ? 2 : cols_needed <= 32 ? 4 : 8; }

// MMA column groups of a routed call. The tile kernels split an expert's
// pairs into runs of 8 * NT, so one group serves any routing; two pay off
// only when experts average more than 8 pairs (fewer weight re-reads).
static int routed_nt(int npairs, int E) {
  const int distinct = std::max(1, std::min(E, npairs));
  return (npairs + distinct - 1) / distinct > 8 ? 2 : 1;
}

// Upper bound on the tile kernels' run count (distinct experts plus splits).
static int route_runs_max(int npairs, int E, int NT) {
  return std::min(npairs, std::min(E, npairs) + npairs / (8 * NT));
}

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
static int occupancy_grid(K kernel, size_t smem, int items, int num_sms) {
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
  const int want = (items + kDecodeWarps - 1) / kDecodeWarps;
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

// The prep kernel as a programmatic dependent of whatever precedes it on the
// stream (the previous call's last kernel triggers early); it waits before
// its first read or write.
static int launch_prep(int blocks, cudaStream_t st, const uint16_t* x, int T, int cols, uint16_t* xp, int32_t* zero,
                       int nzero, const int32_t* ids, int npairs, int E, int32_t* status,
                       const PrepStage& sg = PrepStage{}) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute at[1] = {pdl_attr()};
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_prep, x, T, cols, xp, zero, nzero, ids, npairs, E, status, sg) == cudaSuccess ? 0
                                                                                                               : -4;
}

// Zeroes n words and the floor's timeout flag after the preceding kernel
// completes (programmatic dependent, like the prep kernel; its dependents
// launch only after that wait).
__global__ void __launch_bounds__(256) k_zero(uint32_t* __restrict__ out, size_t n) {
  griddep_wait();
  griddep_launch();
  if (blockIdx.x == 0 && threadIdx.x == 0) g_floor_status = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) out[i] = 0u;
}

// out[i] = bf16_rn(in[i]): the last step of an expert-parallel decode, after
// the ranks' float32 partials are summed.
__global__ void __launch_bounds__(256) k_to_bf16(const float* __restrict__ in, uint16_t* __restrict__ out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = f32_to_bf16_bits(in[i]);
}

int launch_to_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t st, int num_sms) {
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 8));
  k_to_bf16<<<(unsigned)blocks, 256, 0, st>>>(in, out, n);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

GemvWs gemv_ws(int T, int rows, int cols) {
  GemvWs ws;
  const int tiles = (rows + kTile - 1) / kTile;
  const int S = (cols / 256) / item_blocks(cols);
  const int nc = 8 * nt_for(T);
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.xperm = o;
  o = align256(o + (size_t)T * cols * 2);
  ws.cnt = o;
  o = align256(o + (size_t)tiles * 4);
  ws.part = o;
  o = align256(o + (S > 1 ? (size_t)tiles * S * nc * kTile * 4 : 0));
  ws.total = o;
  return ws;
}

template <int MODE, int F0, int F1, int NT, bool BSM>
static int launch_stream(const CUtensorMap& m0, const CUtensorMap& m1, const UnitArgs& a, int items, cudaStream_t st,
                         int num_sms, bool pdl) {
  auto kern = k_stream<MODE, F0, F1, NT, BSM>;
  // the item-index dividers follow this launch's own geometry
  UnitArgs args = a;
  args.wait_ns = g_wait_ns.load();
  args.expire = g_expire.load();
  args.div_s = FastDiv::of((uint32_t)a.splits);
  args.div_tiles = FastDiv::of((uint32_t)((a.w0.rows + kTile - 1) / kTile));
  const size_t smem = stream_smem<F0, F1>(a.w0.cols, BSM ? a.act_rows : 0);
  if (set_smem(kern, smem)) return -4;
  const int grid = occupancy_grid(kern, smem, items, num_sms);
  if (grid < 0) return -4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1] = {pdl_attr()};
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, m0, m1, args) == cudaSuccess ? 0 : -4;
}

template <int MODE, int F0, int F1, int NT, bool BSM>
static int launch_tiles(const CUtensorMap& m0, const CUtensorMap& m1, const UnitArgs& a, int groups, cudaStream_t st,
                        int num_sms, bool pdl) {
  auto kern = k_tiles<MODE, F0, F1, NT, BSM>;
  UnitArgs args = a;
  args.wait_ns = g_wait_ns.load();
  args.expire = g_expire.load();
  args.div_s = FastDiv::of((uint32_t)a.splits);
  const int tiles = (a.w0.rows + kTile - 1) / kTile;
  args.div_tiles = FastDiv::of((uint32_t)(MODE == MODE_SWITCH ? (tiles + a.tpg - 1) / a.tpg : tiles));
  const size_t smem = tiles_smem<MODE, F0, F1, NT>(a.w0.cols, a.T, a.T * a.topk, BSM ? a.act_rows : 0);
  if (set_smem(kern, smem)) return -4;
  KernelCache* kc = kcache(reinterpret_cast<const void*>(kern));
  int per_sm = 0;
  if (kc && kc->occ_smem == smem) {
    per_sm = kc->occ;
  } else {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeWarps * 32, smem) != cudaSuccess) return -4;
    if (kc) {
      kc->occ_smem = smem;
      kc->occ = per_sm;
    }
  }
  if (per_sm < 1) return -4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::max(1, std::min(groups, per_sm * num_sms)));
  cfg.blockDim = dim3(kDecodeWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1] = {pdl_attr()};
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, m0, m1, args) == cudaSuccess ? 0 : -4;
}

// Activation rows a stream launch can keep in shared memory (0: read them
// through the read-only path instead).
static int act_rows_smem(int NT, int rows_needed, int cols) {
  if (NT != 1) return 0;
  return (size_t)rows_needed * (cols / 64 * 80) * 2 <= kActSmemMax ? rows_needed : 0;
}

static void split_args(UnitArgs& a, int cols) {
  a.bpi = item_blocks(cols);
  a.splits = (cols / 256) / a.bpi;
  a.async_sc = async_scales(cols) ? 1 : 0;
}

template <int MODE, int F0, int F1, int NT>
static int launch_stream_any(const CUtensorMap& m0, const CUtensorMap& m1, UnitArgs a, int items, cudaStream_t st,
                             int num_sms, bool pdl, int act_rows) {
  if constexpr (NT == 1) {
    if (act_rows > 0) {
      a.act_rows = act_rows;
      return launch_stream<MODE, F0, F1, NT, true>(m0, m1, a, items, st, num_sms, pdl);
    }
  }
  a.act_rows = 0;
  return launch_stream<MODE, F0, F1, NT, false>(m0, m1, a, items, st, num_sms, pdl);
}

template <int FMT, int NT>
static int gemv_impl(const WDev& w, int expert, const Values& V, const uint16_t* x, int T, float* y, char* ws,
                     cudaStream_t st, int num_sms, bool tiles_ok) {
  const GemvWs L = gemv_ws(T, w.rows, w.cols);
  UnitArgs a = {};
  split_args(a, w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, a.bpi)) return -4;
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  const int tiles = (w.rows + kTile - 1) / kTile;
  if constexpr (NT == 1) {
    // A tall matrix with up to 4 tokens: the switch tile kernel with every
    // pair on `expert` (no ids array). One launch, the call's first: x rows
    // in shared memory, each CTA sums a tile group's slices in its own
    // shared memory (no prep kernel, no device-wide counters). Items of two
    // blocks (half the usual 16-row x 1024-weight slice where rows have a
    // multiple of four blocks): one tile per CTA, twice the CTAs, half the
    // decode per warp; the scales then come from the planes, since the
    // images hold four-block slices. 2048x4096 at one token: 4.75 against
    // 5.57 us with four-block items and 7.4 us on the stream kernel; small
    // matrices stay on the stream kernel.
    if (tiles_ok && T <= 4 && tiles >= 64 && act_rows_smem(1, T, w.cols)) {
      CUtensorMap map2 = map;
      if (a.bpi == 4) {
        a.bpi = 2;
        a.splits *= 2;
        if (make_qs_map(&map2, w, a.bpi)) return -4;
      }
      UnitArgs b = a;
      b.first = 1;
      b.check_ids = 0;
      b.w0 = w;
      b.w1 = w;
      if (b.bpi != item_blocks(w.cols)) b.w0.slots = b.w1.slots = nullptr;
      b.V = V;
      b.ids = nullptr;
      b.expert = expert;
      b.act = xp;
      b.xraw = x;
      b.T = T;
      b.topk = 1;
      b.yf = y;
      b.status = status;
      b.act_rows = T;
      b.tpg = std::max(1, kDecodeWarps / b.splits);
      return launch_tiles<MODE_SWITCH, FMT, FMT, 1, true>(map2, map2, b, (tiles + b.tpg - 1) / b.tpg, st, num_sms,
                                                          true);
    }
  }
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * (w.cols / 16) + 63) / 64)));
  const int nzero = (int)((L.part - L.cnt) / 4);  // the tile counters
  if (launch_prep(pblocks, st, x, T, w.cols, xp, cnt, nzero, nullptr, 0, 1, status)) return -4;
  a.w0 = w;
  a.w1 = w;
  a.V = V;
  a.act = xp;
  a.xraw = x;
  a.T = T;
  a.topk = 1;
  a.expert = expert;
  a.yf = y;
  a.cnt = cnt;
  a.part = reinterpret_cast<float*>(ws + L.part);
  a.status = status;
  return launch_stream_any<MODE_GEMV, FMT, FMT, NT>(map, map, a, tiles * a.splits, st, num_sms, true,
                                                    act_rows_smem(NT, T, w.cols));
}

int launch_gemv(const WDev& w, int fmt, int expert, const Values& V, const uint16_t* x, int T, float* y, char* ws,
                cudaStream_t st, int num_sms, bool tiles_ok) {
  const int NT = nt_for(T);
#define IQK_GEMV(F, N) \
  if (fmt == F && NT == N) return gemv_impl<F, N>(w, expert, V, x, T, y, ws, st, num_sms, tiles_ok);
  IQK_GEMV(FMT_KS, 1) IQK_GEMV(FMT_KS, 2) IQK_GEMV(FMT_KS, 4) IQK_GEMV(FMT_KS, 8)
  IQK_GEMV(FMT_K, 1) IQK_GEMV(FMT_K, 2) IQK_GEMV(FMT_K, 4) IQK_GEMV(FMT_K, 8)
#undef IQK_GEMV
  return -3;
}

DecodeWs decode_ws(int T, int topk, int experts, int hidden, int inter) {
  DecodeWs ws;
  const int npairs = T * topk;
  (void)experts;
  ws.c2 = chunking(inter, hidden);
  ws.c3 = chunking(hidden, inter);
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.xperm = o;
  o = align256(o + (size_t)T * hidden * 2);
  ws.hperm = o;
  o = align256(o + (size_t)npairs * inter * 2);
  ws.ready = o;
  o = align256(o + (size_t)npairs * 4);
  ws.hin = o;  // ids and p copied from host memory
  o = align256(o + (size_t)npairs * 8);
  ws.total = o;
  return ws;
}

template <int FG, int FU, int FD, int NT>
static int decode_impl(const WDev& g, const WDev& u, const WDev& d, const Values& V, const uint16_t* x, int T,
                       const int32_t* ids, const float* p, int topk, uint16_t* y, float* yf, int ebase, char* ws,
                       cudaStream_t st, int num_sms, bool host_io) {
  static_assert(NT == 1 || NT == 2, "routed decode: one or two MMA column groups");
  const DecodeWs L = decode_ws(T, topk, g.experts, g.cols, g.rows);
  const int npairs = T * topk;
  UnitArgs a = {};
  split_args(a, g.cols);
  CUtensorMap mg, mu, md;
  if (make_qs_map(&mg, g, a.bpi) || make_qs_map(&mu, u, a.bpi) || make_qs_map(&md, d, item_blocks(d.cols))) return -4;
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  uint16_t* hp = reinterpret_cast<uint16_t*>(ws + L.hperm);
  const int ar = act_rows_smem(NT, T, g.cols);  // x rows in shared memory, else transposed by the prep kernel
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * (g.cols / 16) + 63) / 64)));
  // a shard skips the ids of other shards silently, so it checks none
  const bool shard = yf != nullptr;
  // h rows in the down kernel's shared memory: it takes each run of pairs as
  // soon as the run's h is complete (per-run counters, zeroed by the prep
  // kernel). Otherwise, with x staged in shared memory there is nothing to
  // prepare: the gate/up kernel is the call's first kernel and resets the
  // status word itself.
  const int hrows = act_rows_smem(NT, npairs, d.cols);
  int32_t* ready = hrows ? reinterpret_cast<int32_t*>(ws + L.ready) : nullptr;
  // Host-resident inputs: the prep kernel reads each input byte once over the
  // host link into the workspace (x as it is where its rows are staged in
  // shared memory, else slot-transposed as usual), and the tile kernels read
  // the copies after waiting for it. y is written to host memory directly.
  PrepStage sg = {};
  const int32_t* ids_k = ids;
  const float* p_k = p;
  const uint16_t* x_k = x;
  if (host_io) {
    int32_t* ids_s = reinterpret_cast<int32_t*>(ws + L.hin);
    float* p_s = reinterpret_cast<float*>(ws + L.hin + (size_t)npairs * 4);
    sg.ids = ids;
    sg.p = p;
    sg.ids_out = ids_s;
    sg.p_out = p_s;
    sg.n = npairs;
    if (ar) {
      sg.xraw = reinterpret_cast<const uint4*>(x);
      sg.xraw_out = reinterpret_cast<uint4*>(xp);
      sg.nx = T * g.cols / 8;
      x_k = xp;
    }
    ids_k = ids_s;
    p_k = p_s;
  }
  if ((!ar || ready || host_io) && launch_prep(ar ? 1 : pblocks, st, x, ar ? 0 : T, g.cols, xp, ready,
                                               ready ? npairs : 0, ids, shard ? 0 : npairs, g.experts, status, sg))
    return -4;
  a.first = (ar && !ready && !host_io) ? 1 : 0;
  a.wait_in = host_io ? 1 : 0;
  a.ready = ready;
  a.check_ids = shard ? 0 : 1;
  a.ebase = ebase;
  a.w0 = g;
  a.w1 = u;
  a.V = V;
  a.ids = ids_k;
  a.p = p_k;
  a.act = xp;
  a.xraw = x_k;
  a.T = T;
  a.topk = topk;
  a.out16 = hp;
  a.status = status;
  a.act_rows = ar;
  const int groups = route_runs_max(npairs, g.experts, NT) * L.c2.tiles;
  const int rc = ar ? launch_tiles<MODE_GATEUP, FG, FU, NT, true>(mg, mu, a, groups, st, num_sms, true)
                    : launch_tiles<MODE_GATEUP, FG, FU, NT, false>(mg, mu, a, groups, st, num_sms, true);
  if (rc) return rc;
  UnitArgs b = a;
  b.first = 0;
  split_args(b, d.cols);
  b.w0 = d;
  b.w1 = d;
  b.act = hp;
  b.out16 = y;
  b.yf = yf;
  b.act_rows = hrows;
  return b.act_rows ? launch_tiles<MODE_DOWN, FD, FD, NT, true>(md, md, b, L.c3.tiles, st, num_sms, true)
                    : launch_tiles<MODE_DOWN, FD, FD, NT, false>(md, md, b, L.c3.tiles, st, num_sms, true);
}

int launch_moe_decode(const WDev& g, int fg, const WDev& u, int fu, const WDev& d, int fd, const Values& V,
                      const uint16_t* x, int T, const int32_t* ids, const float* p, int topk, uint16_t* y, float* yf,
                      int ebase, char* ws, cudaStream_t st, int num_sms, bool host_io) {
  const int NT = routed_nt(T * topk, g.experts);
  const int key = fg * 4 + fu * 2 + fd;
#define IQK_DEC(G, U, D, N)                  \
  if (key == G * 4 + U * 2 + D && NT == N) \
    return decode_impl<G, U, D, N>(g, u, d, V, x, T, ids, p, topk, y, yf, ebase, ws, st, num_sms, host_io);
#define IQK_DEC_N(G, U, D) IQK_DEC(G, U, D, 1) IQK_DEC(G, U, D, 2)
  IQK_DEC_N(0, 0, 0) IQK_DEC_N(0, 0, 1) IQK_DEC_N(0, 1, 0) IQK_DEC_N(0, 1, 1)
  IQK_DEC_N(1, 0, 0) IQK_DEC_N(1, 0, 1) IQK_DEC_N(1, 1, 0) IQK_DEC_N(1, 1, 1)
#undef IQK_DEC_N
#undef IQK_DEC
  return -3;
}

SwitchWs switch_ws(int T, int topk, int experts, int rows, int cols) {
  SwitchWs ws;
  (void)topk;
  (void)experts;
  (void)rows;
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.xperm = o;
  o = align256(o + (size_t)T * cols * 2);
  ws.total = o;
  return ws;
}

template <int FMT, int NT>
static int switch_impl(const WDev& w, const Values& V, const uint16_t* x, int T, const int32_t* ids, int topk,
                       float* y, char* ws, cudaStream_t st, int num_sms) {
  static_assert(NT == 1 || NT == 2, "switch decode: one or two MMA column groups");
  const SwitchWs L = switch_ws(T, topk, w.experts, w.rows, w.cols);
  const int npairs = T * topk;
  UnitArgs a = {};
  split_args(a, w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, a.bpi)) return -4;
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  const int tiles = (w.rows + kTile - 1) / kTile;
  const int ar = act_rows_smem(NT, T, w.cols);  // x rows in shared memory, else transposed by the prep kernel
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * (w.cols / 16) + 63) / 64)));
  // as in the routed decode: with x in shared memory the tile kernel is the call's first kernel
  if (!ar && launch_prep(pblocks, st, x, T, w.cols, xp, nullptr, 0, ids, npairs, w.experts, status)) return -4;
  a.first = ar ? 1 : 0;
  a.check_ids = 1;
  a.w0 = w;
  a.w1 = w;
  a.V = V;
  a.ids = ids;
  a.act = xp;
  a.xraw = x;
  a.T = T;
  a.topk = topk;
  a.yf = y;
  a.status = status;
  a.act_rows = ar;
  // a group is tpg tiles of one run, splits * tpg <= warps items
  a.tpg = std::max(1, kDecodeWarps / a.splits);
  const int groups = route_runs_max(npairs, w.experts, NT) * ((tiles + a.tpg - 1) / a.tpg);
  return ar ? launch_tiles<MODE_SWITCH, FMT, FMT, NT, true>(map, map, a, groups, st, num_sms, true)
            : launch_tiles<MODE_SWITCH, FMT, FMT, NT, false>(map, map, a, groups, st, num_sms, true);
}

int launch_switch_decode(const WDev& w, int fmt, const Values& V, const uint16_t* x, int T, const int32_t* ids,
                         int topk, float* y, char* ws, cudaStream_t st, int num_sms) {
  const int NT = routed_nt(T * topk, w.experts);
#define IQK_SW(F, N) \
  if (fmt == F && NT == N) return switch_impl<F, N>(w, V, x, T, ids, topk, y, ws, st, num_sms);
  IQK_SW(FMT_KS, 1) IQK_SW(FMT_KS, 2) IQK_SW(FMT_K, 1) IQK_SW(FMT_K, 2)
#undef IQK_SW
  return -3;
}

size_t slots_bytes(const WDev& w, int fmt) {
  const int bpi = item_blocks(w.cols);
  const int64_t S = (w.cols / 256) / bpi;
  const int64_t tiles = (w.rows + kTile - 1) / kTile;
  const uint32_t sb = fmt == FMT_KS ? Slot<FMT_KS>::bytes(bpi) : Slot<FMT_K>::bytes(bpi);
  return (size_t)((int64_t)w.experts * tiles * S * sb);
}

int launch_pack_slots(const WDev& w, int fmt, uint8_t* out, cudaStream_t st, int num_sms) {
  const int bpi = item_blocks(w.cols);
  const int64_t n = (int64_t)w.experts * ((w.rows + kTile - 1) / kTile) * ((w.cols / 256) / bpi) * kTile;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 8));
  if (fmt == FMT_KS) k_pack_slots<FMT_KS><<<(unsigned)blocks, 256, 0, st>>>(w, bpi, out);
  else k_pack_slots<FMT_K><<<(unsigned)blocks, 256, 0, st>>>(w, bpi, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

int launch_floor(const WDev& w, int fmt, const int32_t* experts, int n, uint32_t* out, cudaStream_t st,
                 int num_sms) {
  UnitArgs a = {};
  split_args(a, w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, a.bpi)) return -4;
  {
    const size_t nw = (size_t)n * w.rows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max<size_t>(1, std::min<size_t>((nw + 255) / 256, (size_t)num_sms)));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute at[1] = {pdl_attr()};
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_zero, out, nw) != cudaSuccess) return -4;
  }
  a.w0 = w;
  a.w1 = w;
  a.elist = experts;
  a.nexp = n;
  a.outx = out;
  a.T = 1;
  a.topk = 1;
  a.status = nullptr;  // the floor reports a timeout through g_floor_status
  const int items = n * ((w.rows + kTile - 1) / kTile) * a.splits;
  if (fmt == FMT_KS) return launch_stream<MODE_FLOOR, FMT_KS, FMT_KS, 1, false>(map, map, a, items, st, num_sms, true);
  return launch_stream<MODE_FLOOR, FMT_K, FMT_K, 1, false>(map, map, a, items, st, num_sms, true);
}

}  // namespace iqk
