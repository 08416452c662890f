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
  c.nb = (nbk % 4 == 0) ? 4 : ((nbk % 2 == 0) ? 2 : 1);
  c.nkc = nbk / c.nb;
  c.tiles = (rows + kTile - 1) / kTile;
  return c;
}

// ------------------------------------------------------------ row scales
template <int FMT>
struct RowSc;
template <>
struct RowSc<FMT_KS> {
  uint32_t scl[4];
  uint32_t sch, sex;  // byte b = block b of the unit
  float d;
};
template <>
struct RowSc<FMT_K> {
  uint32_t scl[8];
  uint32_t sex[4];  // low 16 bits = block b
  float d[4];
};

template <int FMT>
__device__ __forceinline__ void load_row_scales(RowSc<FMT>& s, const WDev& w, int64_t er, bool valid,
                                                int kb0, int nb) {
  if constexpr (FMT == FMT_KS) {
    s.sch = 0;
    s.sex = 0;
    s.d = 0.f;
#pragma unroll
    for (int b = 0; b < 4; b++) s.scl[b] = 0;
    if (valid) {
      const int64_t base = er * (w.cols / 256) + kb0;
#pragma unroll
      for (int b = 0; b < 4; b++) {
        if (b < nb) {
          s.scl[b] = __ldg(w.scl + base + b);
          s.sch |= (uint32_t)__ldg(w.sch + base + b) << (8 * b);
          s.sex |= (uint32_t)__ldg(reinterpret_cast<const uint8_t*>(w.sex) + base + b) << (8 * b);
        }
      }
      s.d = __half2float(__ushort_as_half(__ldg(w.dv + er)));
    }
  } else {
#pragma unroll
    for (int b = 0; b < 8; b++) s.scl[b] = 0;
#pragma unroll
    for (int b = 0; b < 4; b++) {
      s.sex[b] = 0;
      s.d[b] = 0.f;
    }
    if (valid) {
      const int64_t sb = er * (w.cols / 128) + 2 * kb0;
      const int64_t xb = er * (w.cols / 256) + kb0;
#pragma unroll
      for (int b = 0; b < 4; b++) {
        if (b < nb) {
          s.scl[2 * b] = __ldg(w.scl + sb + 2 * b);
          s.scl[2 * b + 1] = __ldg(w.scl + sb + 2 * b + 1);
          s.sex[b] = __ldg(reinterpret_cast<const uint16_t*>(w.sex) + xb + b);
          s.d[b] = __half2float(__ushort_as_half(__ldg(w.dv + xb + b)));
        }
      }
    }
  }
}

// Table index of the sub-blocks covering words 4t..4t+3 of block b.
// IQ2_KS: (low4 | high<<4) + 32*alphabet, words (4t, 4t+1) in sub-block 2t.
// IQ2_K:  nibble + 16*alphabet, word 4t+m is sub-block 4t+m.
template <int FMT>
__device__ __forceinline__ void combos(const RowSc<FMT>& s, int b, int t, uint32_t (&c)[4]) {
  if constexpr (FMT == FMT_KS) {
    const uint32_t sb = (s.scl[b] >> (8 * t)) & 0xFFu;
    const uint32_t hb = (s.sch >> (8 * b + 2 * t)) & 3u;
    const uint32_t ab = (s.sex >> (8 * b + 2 * t)) & 3u;
    const uint32_t c0 = (sb & 15u) | ((hb & 1u) << 4) | ((ab & 1u) << 5);
    const uint32_t c1 = (sb >> 4) | ((hb >> 1) << 4) | ((ab >> 1) << 5);
    c[0] = c0;
    c[1] = c0;
    c[2] = c1;
    c[3] = c1;
  } else {
    const uint32_t sw = s.scl[2 * b + (t >> 1)] >> (16 * (t & 1));
    const uint32_t x = (s.sex[b] >> (4 * t)) & 15u;
#pragma unroll
    for (int m = 0; m < 4; m++) c[m] = ((sw >> (4 * m)) & 15u) | (((x >> m) & 1u) << 4);
  }
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

// One 16-row tile over nb blocks: acc[n] += W(16 x k) * B(k x 8 columns of group n).
// sq: the tile's qs in shared memory, row stride ldw words. bsrc[n]: this
// lane's activation column (slot-transposed layout) or nullptr for a zero column.
template <int FMT, int NT>
__device__ __forceinline__ void tile_mma(const uint32_t* __restrict__ sq, int ldw, int nb, int kb0,
                                         const RowSc<FMT>& sg, const RowSc<FMT>& sh,
                                         const uint2* __restrict__ lut, const uint16_t* const (&bsrc)[NT],
                                         float (&acc)[NT][4], int g, int t) {
#pragma unroll
  for (int b = 0; b < 4; b++) {
    if (b >= nb) break;
    const uint4 qg = *reinterpret_cast<const uint4*>(sq + g * ldw + b * 16 + 4 * t);
    const uint4 qh = *reinterpret_cast<const uint4*>(sq + (g + 8) * ldw + b * 16 + 4 * t);
    const uint32_t qgv[4] = {qg.x, qg.y, qg.z, qg.w};
    const uint32_t qhv[4] = {qh.x, qh.y, qh.z, qh.w};
    uint32_t cg[4], ch[4];
    combos<FMT>(sg, b, t, cg);
    combos<FMT>(sh, b, t, ch);
    float fr[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) fr[n][e] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; m++) {
      const uint2 tg = lut[cg[m]];
      const uint2 th = lut[ch[m]];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const Pair2 pg = lookup_slot(qgv[m], i, tg.x, tg.y);
        const Pair2 ph = lookup_slot(qhv[m], i, th.x, th.y);
        const int off = 256 * (kb0 + b) + 64 * t + 16 * m + 4 * i;
#pragma unroll
        for (int n = 0; n < NT; n++) {
          uint2 bv = make_uint2(0u, 0u);
          if (bsrc[n] != nullptr) bv = ld_nc_u2(bsrc[n] + off);
          if constexpr (FMT == FMT_K) {
            mma_bf16(fr[n], pg.lo, ph.lo, pg.hi, ph.hi, bv.x, bv.y);
          } else {
            mma_bf16(acc[n], pg.lo, ph.lo, pg.hi, ph.hi, bv.x, bv.y);
          }
        }
      }
    }
    if constexpr (FMT == FMT_K) {
#pragma unroll
      for (int n = 0; n < NT; n++) {
        acc[n][0] = fmaf(sg.d[b], fr[n][0], acc[n][0]);
        acc[n][1] = fmaf(sg.d[b], fr[n][1], acc[n][1]);
        acc[n][2] = fmaf(sh.d[b], fr[n][2], acc[n][2]);
        acc[n][3] = fmaf(sh.d[b], fr[n][3], acc[n][3]);
      }
    }
  }
  if constexpr (FMT == FMT_KS) {
#pragma unroll
    for (int n = 0; n < NT; n++) {
      acc[n][0] *= sg.d;
      acc[n][1] *= sg.d;
      acc[n][2] *= sh.d;
      acc[n][3] *= sh.d;
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

__device__ RouteView carve_route(uint8_t* p, int n) {
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

__device__ void build_route(const int32_t* __restrict__ ids, int n, int E, RouteView r) {
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
  if (tid == 0) {
    int bad = 0;
    for (int p = 0; p < npairs; p++) bad |= (ids[p] < 0 || ids[p] >= E);
    status[0] = bad ? 1 : 0;
  }
  const int64_t n = (int64_t)T * cols;
  for (int64_t e = tid; e < n; e += nth) {
    const int64_t t = e / cols;
    const int k = (int)(e - t * cols);
    xp[t * cols + perm16(k)] = x[e];
  }
}

// ---------------------------------------------------------- shared pieces
struct WarpRing {
  uint32_t* stage;  // [kStages][mats][16][ldw]
  uint64_t* bar;    // [kStages]
  int stage_words;  // mats * 16 * ldw
};

__device__ __forceinline__ bool wait_stage(WarpRing& ring, int s, uint32_t par, int32_t* status) {
  if (mbar_wait_bounded(&ring.bar[s], par)) return true;
  if ((threadIdx.x & 31) == 0) atomicOr(status, 2);
  return false;
}

// After a wait gave up: wait (bounded) for every stage still in flight so no
// copy lands in shared memory after the CTA exits.
__device__ void drain_ring(WarpRing& ring, const uint32_t* issued_phase, int nstages) {
  for (int s = 0; s < nstages; s++) {
    if (issued_phase[s] != 0xFFFFFFFFu) (void)mbar_wait_bounded(&ring.bar[s], issued_phase[s]);
  }
}

// --------------------------------------------------------------- GEMV
template <int FMT, int NT>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_gemv(const __grid_constant__ CUtensorMap map, WDev w,
                                                            int expert, Values V, const uint16_t* __restrict__ xp,
                                                            int T, float* __restrict__ y, int32_t* __restrict__ cnt,
                                                            float* __restrict__ part, int32_t* __restrict__ status,
                                                            Chunking c) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ldw = c.nb * 16;
  const int stage_words = kTile * ldw;
  uint32_t* stages = reinterpret_cast<uint32_t*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kDecodeWarps * kStages * stage_words * 4);
  uint2* lut = reinterpret_cast<uint2*>(bars + kDecodeWarps * kStages);
  build_lut<FMT>(lut, V);
  WarpRing ring{stages + (size_t)wid * kStages * stage_words, bars + wid * kStages, stage_words};
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&ring.bar[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int nunits = c.tiles * c.nkc;
  const int W = gridDim.x * kDecodeWarps;
  const int gw = blockIdx.x * kDecodeWarps + wid;
  uint32_t issued[kStages];
  auto issue = [&](int it, int s) {
    const int id = gw + it * W;
    issued[s] = 0xFFFFFFFFu;
    if (id >= nunits) return;
    issued[s] = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc, tile = id / c.nkc;
    if (lane == 0) {
      mbar_arrive_expect_tx(&ring.bar[s], (uint32_t)stage_words * 4);
      tma_load_2d(ring.stage + (size_t)s * stage_words, &map, kc * ldw, expert * w.rows + tile * kTile,
                  &ring.bar[s]);
    }
  };
  for (int s = 0; s < kStages; s++) issue(s, s);
  griddep_wait();
  for (int it = 0;; it++) {
    const int id = gw + it * W;
    if (id >= nunits) break;
    const int s = it % kStages;
    const uint32_t par = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc, tile = id / c.nkc;
    const int rg = tile * kTile + g, rh = rg + 8;
    RowSc<FMT> sg, sh;
    load_row_scales<FMT>(sg, w, (int64_t)expert * w.rows + rg, rg < w.rows, kc * c.nb, c.nb);
    load_row_scales<FMT>(sh, w, (int64_t)expert * w.rows + rh, rh < w.rows, kc * c.nb, c.nb);
    const uint16_t* bsrc[NT];
#pragma unroll
    for (int n = 0; n < NT; n++) {
      const int col = 8 * n + g;
      bsrc[n] = col < T ? xp + (size_t)col * w.cols : nullptr;
    }
    if (!wait_stage(ring, s, par, status)) {
      drain_ring(ring, issued, kStages);
      return;
    }
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) acc[n][e] = 0.f;
    tile_mma<FMT, NT>(ring.stage + (size_t)s * stage_words, ldw, c.nb, kc * c.nb, sg, sh, lut, bsrc, acc, g, t);
    __syncwarp();
    issue(it + kStages, s);
    if (c.nkc == 1) {
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int col = 8 * n + 2 * t + (e & 1);
          const int row = tile * kTile + g + 8 * (e >> 1);
          if (col < T && row < w.rows) y[(size_t)col * w.rows + row] = acc[n][e];
        }
      continue;
    }
    // partial slot [tile][kc][col][16]
    float* slot = part + ((size_t)tile * c.nkc + kc) * (8 * NT) * kTile;
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const int col = 8 * n + 2 * t + (e & 1);
        const int r = g + 8 * (e >> 1);
        slot[col * kTile + r] = acc[n][e];
      }
    __threadfence();
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = atomicAdd(cnt + tile, 1);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != c.nkc - 1) continue;
    __threadfence();
    const float* base = part + (size_t)tile * c.nkc * (8 * NT) * kTile;
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const int col = 8 * n + 2 * t + (e & 1);
        const int r = g + 8 * (e >> 1);
        const int row = tile * kTile + r;
        if (col >= T || row >= w.rows) continue;
        float sum = 0.f;
        for (int k = 0; k < c.nkc; k++) sum += __ldcg(base + ((size_t)k * (8 * NT) + col) * kTile + r);
        y[(size_t)col * w.rows + row] = sum;
      }
  }
}

// ------------------------------------------------------ gate/up + SwiGLU
template <int FG, int FU, int NT>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_gateup(
    const __grid_constant__ CUtensorMap mg, const __grid_constant__ CUtensorMap mu, WDev wg, WDev wu,
    Values V, const int32_t* __restrict__ ids, int T, int topk, const uint16_t* __restrict__ xp,
    uint16_t* __restrict__ hp, int32_t* __restrict__ cnt, float* __restrict__ part,
    int32_t* __restrict__ status, Chunking c) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ldw = c.nb * 16;
  const int mat_words = kTile * ldw;
  const int stage_words = 2 * mat_words;
  const int npairs = T * topk;
  const int F = wg.rows, H = wg.cols;
  uint32_t* stages = reinterpret_cast<uint32_t*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kDecodeWarps * kStages * stage_words * 4);
  uint2* lut_g = reinterpret_cast<uint2*>(bars + kDecodeWarps * kStages);
  uint2* lut_u = lut_g + 64;
  RouteView rt = carve_route(reinterpret_cast<uint8_t*>(lut_u + 64), npairs);
  build_lut<FG>(lut_g, V);
  build_lut<FU>(lut_u, V);
  WarpRing ring{stages + (size_t)wid * kStages * stage_words, bars + wid * kStages, stage_words};
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&ring.bar[s], 1);
    fence_mbar_init();
  }
  build_route(ids, npairs, wg.experts, rt);  // ends with __syncthreads
  const int D = rt.scalars[0];
  const int nunits = D * c.tiles * c.nkc;
  const int W = gridDim.x * kDecodeWarps;
  const int gw = blockIdx.x * kDecodeWarps + wid;
  uint32_t issued[kStages];
  auto issue = [&](int it, int s) {
    const int id = gw + it * W;
    issued[s] = 0xFFFFFFFFu;
    if (id >= nunits) return;
    issued[s] = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc;
    const int rest = id / c.nkc;
    const int tile = rest % c.tiles, u = rest / c.tiles;
    const int e = rt.uexp[u];
    if (lane == 0) {
      uint32_t* st = ring.stage + (size_t)s * stage_words;
      mbar_arrive_expect_tx(&ring.bar[s], (uint32_t)stage_words * 4);
      tma_load_2d(st, &mg, kc * ldw, e * wg.rows + tile * kTile, &ring.bar[s]);
      tma_load_2d(st + mat_words, &mu, kc * ldw, e * wu.rows + tile * kTile, &ring.bar[s]);
    }
  };
  for (int s = 0; s < kStages; s++) issue(s, s);
  griddep_launch();
  griddep_wait();
  for (int it = 0;; it++) {
    const int id = gw + it * W;
    if (id >= nunits) break;
    const int s = it % kStages;
    const uint32_t par = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc;
    const int rest = id / c.nkc;
    const int tile = rest % c.tiles, u = rest / c.tiles;
    const int e = rt.uexp[u];
    const int p0 = rt.ustart[u], ncols = rt.ustart[u + 1] - p0;
    const int rg = tile * kTile + g, rh = rg + 8;
    RowSc<FG> sgg, sgh;
    RowSc<FU> sug, suh;
    load_row_scales<FG>(sgg, wg, (int64_t)e * F + rg, rg < F, kc * c.nb, c.nb);
    load_row_scales<FG>(sgh, wg, (int64_t)e * F + rh, rh < F, kc * c.nb, c.nb);
    load_row_scales<FU>(sug, wu, (int64_t)e * F + rg, rg < F, kc * c.nb, c.nb);
    load_row_scales<FU>(suh, wu, (int64_t)e * F + rh, rh < F, kc * c.nb, c.nb);
    const uint16_t* bsrc[NT];
#pragma unroll
    for (int n = 0; n < NT; n++) {
      const int col = 8 * n + g;
      bsrc[n] = col < ncols ? xp + (size_t)(rt.sorted[p0 + col] / topk) * H : nullptr;
    }
    if (!wait_stage(ring, s, par, status)) {
      drain_ring(ring, issued, kStages);
      return;
    }
    float ag[NT][4], au[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) ag[n][q] = au[n][q] = 0.f;
    const uint32_t* st = ring.stage + (size_t)s * stage_words;
    tile_mma<FG, NT>(st, ldw, c.nb, kc * c.nb, sgg, sgh, lut_g, bsrc, ag, g, t);
    tile_mma<FU, NT>(st + mat_words, ldw, c.nb, kc * c.nb, sug, suh, lut_u, bsrc, au, g, t);
    __syncwarp();
    issue(it + kStages, s);
    const int slot_cols = 8 * NT;
    if (c.nkc > 1) {
      const size_t ut = (size_t)u * c.tiles + tile;
      float* slot = part + ((ut * c.nkc + kc) * 2) * slot_cols * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const int col = 8 * n + 2 * t + (q & 1);
          const int r = g + 8 * (q >> 1);
          slot[col * kTile + r] = ag[n][q];
          slot[(slot_cols + col) * kTile + r] = au[n][q];
        }
      __threadfence();
      __syncwarp();
      int prev = 0;
      if (lane == 0) prev = atomicAdd(cnt + ut, 1);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != c.nkc - 1) continue;
      __threadfence();
      const float* base = part + (ut * c.nkc * 2) * slot_cols * kTile;
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const int col = 8 * n + 2 * t + (q & 1);
          const int r = g + 8 * (q >> 1);
          float sg_ = 0.f, su_ = 0.f;
          for (int k = 0; k < c.nkc; k++) {
            const float* sl = base + ((size_t)k * 2) * slot_cols * kTile;
            sg_ += __ldcg(sl + col * kTile + r);
            su_ += __ldcg(sl + (slot_cols + col) * kTile + r);
          }
          ag[n][q] = sg_;
          au[n][q] = su_;
        }
    }
    // SwiGLU and store h in the slot-transposed layout the down kernel reads.
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int col = 8 * n + 2 * t + (q & 1);
        const int f = tile * kTile + g + 8 * (q >> 1);
        if (col >= ncols || f >= F) continue;
        const float gv = ag[n][q], uv = au[n][q];
        const float h = gv / (1.0f + __expf(-gv)) * uv;
        const int pair = rt.sorted[p0 + col];
        hp[(size_t)pair * F + perm16(f)] = f32_to_bf16_bits(h);
      }
  }
}

// ------------------------------------------------------ down + combine
template <int FD, int NT>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_down(
    const __grid_constant__ CUtensorMap md, WDev wd, Values V, const int32_t* __restrict__ ids, int T,
    int topk, const float* __restrict__ p, const uint16_t* __restrict__ hp, uint16_t* __restrict__ y,
    int32_t* __restrict__ cnt, float* __restrict__ part, int32_t* __restrict__ status, Chunking c) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ldw = c.nb * 16;
  const int stage_words = kTile * ldw;
  const int npairs = T * topk;
  const int H = wd.rows, F = wd.cols;
  uint32_t* stages = reinterpret_cast<uint32_t*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kDecodeWarps * kStages * stage_words * 4);
  uint2* lut = reinterpret_cast<uint2*>(bars + kDecodeWarps * kStages);
  RouteView rt = carve_route(reinterpret_cast<uint8_t*>(lut + 64), npairs);
  build_lut<FD>(lut, V);
  WarpRing ring{stages + (size_t)wid * kStages * stage_words, bars + wid * kStages, stage_words};
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&ring.bar[s], 1);
    fence_mbar_init();
  }
  build_route(ids, npairs, wd.experts, rt);
  const int D = rt.scalars[0];
  const int nunits = D * c.tiles * c.nkc;
  const int W = gridDim.x * kDecodeWarps;
  const int gw = blockIdx.x * kDecodeWarps + wid;
  uint32_t issued[kStages];
  auto issue = [&](int it, int s) {
    const int id = gw + it * W;
    issued[s] = 0xFFFFFFFFu;
    if (id >= nunits) return;
    issued[s] = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc;
    const int rest = id / c.nkc;
    const int tile = rest % c.tiles, u = rest / c.tiles;
    if (lane == 0) {
      mbar_arrive_expect_tx(&ring.bar[s], (uint32_t)stage_words * 4);
      tma_load_2d(ring.stage + (size_t)s * stage_words, &md, kc * ldw, rt.uexp[u] * H + tile * kTile,
                  &ring.bar[s]);
    }
  };
  for (int s = 0; s < kStages; s++) issue(s, s);
  griddep_wait();
  if (D == 0) {  // every id was out of range: the block output is zero
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < T * H; i += gridDim.x * blockDim.x) y[i] = 0;
    return;
  }
  for (int it = 0;; it++) {
    const int id = gw + it * W;
    if (id >= nunits) break;
    const int s = it % kStages;
    const uint32_t par = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc;
    const int rest = id / c.nkc;
    const int tile = rest % c.tiles, u = rest / c.tiles;
    const int e = rt.uexp[u];
    const int p0 = rt.ustart[u], ncols = rt.ustart[u + 1] - p0;
    const int rg = tile * kTile + g, rh = rg + 8;
    RowSc<FD> sg, sh;
    load_row_scales<FD>(sg, wd, (int64_t)e * H + rg, rg < H, kc * c.nb, c.nb);
    load_row_scales<FD>(sh, wd, (int64_t)e * H + rh, rh < H, kc * c.nb, c.nb);
    const uint16_t* bsrc[NT];
#pragma unroll
    for (int n = 0; n < NT; n++) {
      const int col = 8 * n + g;
      bsrc[n] = col < ncols ? hp + (size_t)rt.sorted[p0 + col] * F : nullptr;
    }
    if (!wait_stage(ring, s, par, status)) {
      drain_ring(ring, issued, kStages);
      return;
    }
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) acc[n][q] = 0.f;
    tile_mma<FD, NT>(ring.stage + (size_t)s * stage_words, ldw, c.nb, kc * c.nb, sg, sh, lut, bsrc, acc, g, t);
    __syncwarp();
    issue(it + kStages, s);
    // partial per (tile, kc, pair): p * (W_down h)
    float* slab = part + ((size_t)tile * c.nkc + kc) * npairs * kTile;
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int col = 8 * n + 2 * t + (q & 1);
        if (col >= ncols) continue;
        const int pair = rt.sorted[p0 + col];
        slab[(size_t)pair * kTile + g + 8 * (q >> 1)] = __ldg(p + pair) * acc[n][q];
      }
    __threadfence();
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = atomicAdd(cnt + tile, 1);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != c.nkc * D - 1) continue;
    __threadfence();
    // last unit of this tile: y[t][rows] = sum over slots j, then chunks
    for (int o = lane; o < T * kTile; o += 32) {
      const int tok = o / kTile, r = o % kTile;
      const int row = tile * kTile + r;
      if (row >= H) continue;
      float sum = 0.f;
      for (int j = 0; j < topk; j++) {
        const int pair = tok * topk + j;
        if (rt.ids[pair] < 0) continue;
        for (int k = 0; k < c.nkc; k++)
          sum += __ldcg(part + (((size_t)tile * c.nkc + k) * npairs + pair) * kTile + r);
      }
      y[(size_t)tok * H + row] = f32_to_bf16_bits(sum);
    }
  }
}

// ------------------------------------------------------------ floor arm
// Identical loads to the decode kernels (TMA qs tile, per-lane scale loads),
// decode replaced by an XOR fold; every loaded byte reaches the output.
template <int FMT>
__device__ __forceinline__ uint32_t fold_scales(const RowSc<FMT>& s, int kb0, int nb, bool with_row_scale) {
  uint32_t h = 0;
  if constexpr (FMT == FMT_KS) {
#pragma unroll
    for (int b = 0; b < 4; b++) {
      if (b >= nb) break;
      const int kb = kb0 + b;
      h ^= s.scl[b];
      h ^= ((s.sch >> (8 * b)) & 0xFFu) << (8 * (kb & 3));
      h ^= ((s.sex >> (8 * b)) & 0xFFu) << (8 * (kb & 3));
    }
    if (with_row_scale) h ^= (uint32_t)__half_as_ushort(__float2half_rn(s.d));
  } else {
#pragma unroll
    for (int b = 0; b < 4; b++) {
      if (b >= nb) break;
      const int kb = kb0 + b;
      h ^= s.scl[2 * b] ^ s.scl[2 * b + 1];
      h ^= (s.sex[b] & 0xFFFFu) << (16 * (kb & 1));
      h ^= (uint32_t)__half_as_ushort(__float2half_rn(s.d[b])) << (16 * (kb & 1));
    }
  }
  return h;
}

// Timeout flag of the floor arm (it has no workspace); read with
// cudaMemcpyFromSymbol when diagnosing.
__device__ int32_t g_floor_status;

template <int FMT>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_floor(const __grid_constant__ CUtensorMap map, WDev w,
                                                             const int32_t* __restrict__ elist, int nexp,
                                                             uint32_t* __restrict__ out, Chunking c) {
  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* status = &g_floor_status;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ldw = c.nb * 16;
  const int stage_words = kTile * ldw;
  uint32_t* stages = reinterpret_cast<uint32_t*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kDecodeWarps * kStages * stage_words * 4);
  WarpRing ring{stages + (size_t)wid * kStages * stage_words, bars + wid * kStages, stage_words};
  if (lane == 0) {
    for (int s = 0; s < kStages; s++) mbar_init(&ring.bar[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int nunits = nexp * c.tiles * c.nkc;
  const int W = gridDim.x * kDecodeWarps;
  const int gw = blockIdx.x * kDecodeWarps + wid;
  uint32_t issued[kStages];
  auto issue = [&](int it, int s) {
    const int id = gw + it * W;
    issued[s] = 0xFFFFFFFFu;
    if (id >= nunits) return;
    issued[s] = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc;
    const int rest = id / c.nkc;
    const int tile = rest % c.tiles, i = rest / c.tiles;
    if (lane == 0) {
      mbar_arrive_expect_tx(&ring.bar[s], (uint32_t)stage_words * 4);
      tma_load_2d(ring.stage + (size_t)s * stage_words, &map, kc * ldw, elist[i] * w.rows + tile * kTile,
                  &ring.bar[s]);
    }
  };
  for (int s = 0; s < kStages; s++) issue(s, s);
  for (int it = 0;; it++) {
    const int id = gw + it * W;
    if (id >= nunits) break;
    const int s = it % kStages;
    const uint32_t par = (uint32_t)((it / kStages) & 1);
    const int kc = id % c.nkc;
    const int rest = id / c.nkc;
    const int tile = rest % c.tiles, i = rest / c.tiles;
    const int e = elist[i];
    const int rg = tile * kTile + g, rh = rg + 8;
    RowSc<FMT> sg, sh;
    load_row_scales<FMT>(sg, w, (int64_t)e * w.rows + rg, rg < w.rows, kc * c.nb, c.nb);
    load_row_scales<FMT>(sh, w, (int64_t)e * w.rows + rh, rh < w.rows, kc * c.nb, c.nb);
    if (!wait_stage(ring, s, par, status)) {
      drain_ring(ring, issued, kStages);
      return;
    }
    const uint32_t* sq = ring.stage + (size_t)s * stage_words;
    uint32_t hg = 0, hh = 0;
    for (int b = 0; b < c.nb; b++) {
      const uint4 qg = *reinterpret_cast<const uint4*>(sq + g * ldw + b * 16 + 4 * t);
      const uint4 qh = *reinterpret_cast<const uint4*>(sq + (g + 8) * ldw + b * 16 + 4 * t);
      hg ^= qg.x ^ qg.y ^ qg.z ^ qg.w;
      hh ^= qh.x ^ qh.y ^ qh.z ^ qh.w;
    }
    __syncwarp();
    issue(it + kStages, s);
    hg ^= __shfl_xor_sync(0xffffffffu, hg, 1);
    hg ^= __shfl_xor_sync(0xffffffffu, hg, 2);
    hh ^= __shfl_xor_sync(0xffffffffu, hh, 1);
    hh ^= __shfl_xor_sync(0xffffffffu, hh, 2);
    if (t == 0) {
      hg ^= fold_scales<FMT>(sg, kc * c.nb, c.nb, kc == 0);
      hh ^= fold_scales<FMT>(sh, kc * c.nb, c.nb, kc == 0);
      if (rg < w.rows) atomicXor(out + (size_t)i * w.rows + rg, hg);
      if (rh < w.rows) atomicXor(out + (size_t)i * w.rows + rh, hh);
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

static size_t ring_bytes(int mats, int nb) {
  return (size_t)kDecodeWarps * kStages * mats * kTile * nb * 16 * 4 + (size_t)kDecodeWarps * kStages * 8;
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
  per_sm = std::min(per_sm, 2);
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
  const Chunking c = chunking(rows, cols);
  const int NT = nt_for(T);
  GemvWs ws;
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.xperm = o;
  o = align256(o + (size_t)T * cols * 2);
  ws.cnt = o;
  o = align256(o + (size_t)c.tiles * 4);
  ws.part = o;
  o = align256(o + (size_t)c.tiles * c.nkc * 8 * NT * kTile * 4);
  ws.total = o;
  return ws;
}

template <int FMT, int NT>
static int gemv_impl(const WDev& w, int expert, const Values& V, const uint16_t* x, int T, float* y, char* ws,
                     cudaStream_t st, int num_sms) {
  const Chunking c = chunking(w.rows, w.cols);
  const GemvWs L = gemv_ws(T, w.rows, w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, c.nb)) return -4;
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  float* part = reinterpret_cast<float*>(ws + L.part);
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * w.cols + 4095) / 4096)));
  k_prep<<<pblocks, 256, 0, st>>>(x, T, w.cols, xp, cnt, c.tiles, nullptr, 0, 1, status);
  const size_t smem = ring_bytes(1, c.nb) + 64 * 8;
  auto kern = k_gemv<FMT, NT>;
  if (set_smem(kern, smem)) return -4;
  const int grid = occupancy_grid(kern, smem, c.tiles * c.nkc, num_sms);
  if (grid < 0) return -4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1] = {pdl_attr()};
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, map, w, expert, V, (const uint16_t*)xp, T, y, cnt, part, status, c) !=
      cudaSuccess)
    return -4;
  return 0;
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
  if (ws.c2.nkc > 1) o = align256(o + (size_t)ws.dmax * ws.c2.tiles * ws.c2.nkc * 2 * ws.nc * kTile * 4);
  ws.part3 = o;
  o = align256(o + (size_t)ws.c3.tiles * ws.c3.nkc * npairs * kTile * 4);
  ws.total = o;
  return ws;
}

template <int FG, int FU, int FD, int NT>
static int decode_impl(const WDev& g, const WDev& u, const WDev& d, const Values& V, const uint16_t* x, int T,
                       const int32_t* ids, const float* p, int topk, uint16_t* y, char* ws, cudaStream_t st,
                       int num_sms) {
  const DecodeWs L = decode_ws(T, topk, g.experts, g.cols, g.rows);
  const int npairs = T * topk;
  CUtensorMap mg, mu, md;
  if (make_qs_map(&mg, g, L.c2.nb) || make_qs_map(&mu, u, L.c2.nb) || make_qs_map(&md, d, L.c3.nb)) return -4;
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + L.xperm);
  uint16_t* hp = reinterpret_cast<uint16_t*>(ws + L.hperm);
  int32_t* cnt2 = reinterpret_cast<int32_t*>(ws + L.cnt2);
  float* part2 = reinterpret_cast<float*>(ws + L.part2);
  float* part3 = reinterpret_cast<float*>(ws + L.part3);
  // counters for both kernels are contiguous: cnt2 then cnt3
  const int nzero = (int)((L.part2 - L.cnt2) / 4);
  int32_t* cnt3 = reinterpret_cast<int32_t*>(ws + L.cnt3);
  const int pblocks = std::max(1, std::min(num_sms, (int)(((int64_t)T * g.cols + 4095) / 4096)));
  k_prep<<<pblocks, 256, 0, st>>>(x, T, g.cols, xp, cnt2, nzero, ids, npairs, g.experts, status);
  if (cudaGetLastError() != cudaSuccess) return -4;

  const size_t rsm = route_smem_bytes(npairs);
  cudaLaunchAttribute at[1] = {pdl_attr()};
  {
    const size_t smem = ring_bytes(2, L.c2.nb) + 2 * 64 * 8 + rsm;
    auto kern = k_gateup<FG, FU, NT>;
    if (set_smem(kern, smem)) return -4;
    const int grid = occupancy_grid(kern, smem, L.dmax * L.c2.tiles * L.c2.nkc, num_sms);
    if (grid < 0) return -4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecodeWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, mg, mu, g, u, V, ids, T, topk, (const uint16_t*)xp, hp, cnt2, part2, status,
                           L.c2) != cudaSuccess)
      return -4;
  }
  {
    const size_t smem = ring_bytes(1, L.c3.nb) + 64 * 8 + rsm;
    auto kern = k_down<FD, NT>;
    if (set_smem(kern, smem)) return -4;
    const int grid = occupancy_grid(kern, smem, L.dmax * L.c3.tiles * L.c3.nkc, num_sms);
    if (grid < 0) return -4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecodeWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, md, d, V, ids, T, topk, p, (const uint16_t*)hp, y, cnt3, part3, status,
                           L.c3) != cudaSuccess)
      return -4;
  }
  return 0;
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
  const Chunking c = chunking(w.rows, w.cols);
  CUtensorMap map;
  if (make_qs_map(&map, w, c.nb)) return -4;
  if (cudaMemsetAsync(out, 0, (size_t)n * w.rows * 4, st) != cudaSuccess) return -4;
  const size_t smem = ring_bytes(1, c.nb);
  if (fmt == FMT_KS) {
    auto kern = k_floor<FMT_KS>;
    if (set_smem(kern, smem)) return -4;
    const int grid = occupancy_grid(kern, smem, n * c.tiles * c.nkc, num_sms);
    if (grid < 0) return -4;
    kern<<<grid, kDecodeWarps * 32, smem, st>>>(map, w, experts, n, out, c);
  } else {
    auto kern = k_floor<FMT_K>;
    if (set_smem(kern, smem)) return -4;
    const int grid = occupancy_grid(kern, smem, n * c.tiles * c.nkc, num_sms);
    if (grid < 0) return -4;
    kern<<<grid, kDecodeWarps * 32, smem, st>>>(map, w, experts, n, out, c);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
