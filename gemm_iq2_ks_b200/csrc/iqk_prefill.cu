// Prefill path: pairs grouped by expert, each expert's weights dequantized
// once into bfloat16 tensor-core operands and multiplied on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// mlx-iqk 0.1.1 PKG-INFO, section "Surface": a larger call "dequantizes the
// stacked experts in one kernel pass and runs gather_mm, honouring the
// caller's sort flag so each expert's weights are read once per sorted
// prefill". Here the dequantization is not a separate pass: producer warps
// decode the 2-bit codes straight into tensor memory, where the MMA reads
// its A operand.
//
// Launch sequence: grouping (iqk_route.cu) -> gather of token rows in expert
// order -> gate/up grouped GEMM with SwiGLU epilogue -> down grouped GEMM
// (row scale in the epilogue) -> per-token combine, routing-weighted, in slot
// order.
#include <algorithm>

#include "iqk_device.cuh"
#include "iqk_internal.h"
#include "iqk_tc.cuh"

namespace iqk {

constexpr int PF_WARPS = 11;
constexpr int PF_THREADS = PF_WARPS * 32;
constexpr int PF_TMA_WARP = 8;   // qs tiles
constexpr int PF_MMA_WARP = 9;
constexpr int PF_BTMA_WARP = 10;  // token rows (B operand)
constexpr int PF_SA = 2;      // A stages in tensor memory (64 k each)
constexpr int PF_SB = 4;      // B stages in shared memory (64 k each)
constexpr int PF_SQ = 3;      // qs stages in shared memory (256 k each)
// Two CTAs share an SM, each with half of tensor memory (256 columns): two
// 64-column accumulators (pairs per N tile <= 64) and two A stages. The two
// CTAs' pipelines interleave, which hides the long round trip of an A stage
// (decode, store, signal, MMA, commit) better than one deeper pipeline.
constexpr int PF_NMAX = 64;  // pairs per N tile
constexpr uint32_t TM_COLS = 256;
constexpr uint32_t TM_D0 = 0, TM_D1 = 64, TM_A = 128;
constexpr int PF_B_BYTES = PF_NMAX * 128;       // one B stage: 64 rows x 64 bf16
constexpr int PF_Q_BYTES = 2 * 128 * 16 * 4;    // one qs stage: two 128-row tiles x 16 words
constexpr int PF_NBAR = 2 * PF_SQ + 2 * PF_SB + 2 * PF_SA + 2;
constexpr size_t PF_SMEM = (size_t)PF_SB * PF_B_BYTES + (size_t)PF_SQ * PF_Q_BYTES + PF_NBAR * 8 + 2 * 64 * 8 + 64 +
                           1024;  // + alignment slack

struct PfArgs {
  WDev w0, w1;  // gate/up (mode 0) or down/down (mode 1)
  Values V;
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* perm;
  const float* p;
  uint16_t* hs;  // mode 0 output [pairs][inter], slot-transposed along inter
  float* outp;   // mode 1 output [pairs][hidden]
  int32_t* status;
  int E, K, rows, mtiles;
};

// Table entries of one 256-weight block of one row for the producer.
template <int FMT>
struct BlkSc;
template <>
struct BlkSc<FMT_KS> {
  uint32_t scl, sch, sex;
};
template <>
struct BlkSc<FMT_K> {
  uint32_t scl0, scl1, sex;
  float d;
};

template <int FMT>
__device__ __forceinline__ BlkSc<FMT> load_blk(const WDev& w, int64_t grow, int b) {
  BlkSc<FMT> s;
  if constexpr (FMT == FMT_KS) {
    const int64_t i = grow * (w.cols / 256) + b;
    s.scl = __ldg(w.scl + i);
    s.sch = __ldg(w.sch + i);
    s.sex = __ldg(reinterpret_cast<const uint8_t*>(w.sex) + i);
  } else {
    const int64_t i2 = grow * (w.cols / 128) + 2 * b;
    const int64_t i1 = grow * (w.cols / 256) + b;
    s.scl0 = __ldg(w.scl + i2);
    s.scl1 = __ldg(w.scl + i2 + 1);
    s.sex = __ldg(reinterpret_cast<const uint16_t*>(w.sex) + i1);
    s.d = __half2float(__ushort_as_half(__ldg(w.dv + i1)));
  }
  return s;
}

template <int FMT>
__device__ __forceinline__ void build_lut_pf(uint2* lut, const Values& V) {
  if constexpr (FMT == FMT_KS) {
    for (int c = threadIdx.x; c < 64; c += blockDim.x) {
      const float fi = (float)((c & 31) - 16);
      const int a = c >> 5;
      lut[c] = make_uint2(pack_bf16x2(__fmul_rn(fi, a ? V.v[4] : V.v[0]), __fmul_rn(fi, a ? V.v[5] : V.v[1])),
                          pack_bf16x2(__fmul_rn(fi, a ? V.v[6] : V.v[2]), __fmul_rn(fi, a ? V.v[7] : V.v[3])));
    }
  }
}

// The two table words of the sub-block covering word m of chunk cc (0..3)
// inside its 256-block.
// IQ2_KS: bf16(scale_index * value) from the shared table; the row scale d is
//         applied to the accumulator in the epilogue.
// IQ2_K:  bf16_rn((d * float(scale_index)) * value), the page's float32 chain,
//         because d changes every 256 weights along the reduction.
template <int FMT>
__device__ __forceinline__ uint2 table_words(const BlkSc<FMT>& s, int cc, int m, const uint2* lut, const Values& V) {
  if constexpr (FMT == FMT_KS) {
    const int j = 2 * cc + (m >> 1);
    const uint32_t c = ((s.scl >> (4 * j)) & 15u) | (((s.sch >> j) & 1u) << 4) | (((s.sex >> j) & 1u) << 5);
    return lut[c];
  } else {
    const int j = 4 * cc + m;
    const uint32_t w = (j < 8) ? s.scl0 : s.scl1;
    const int idx = (int)((w >> (4 * (j & 7))) & 15u) - 8;
    const int a = (s.sex >> j) & 1;
    const float t = __fmul_rn(s.d, (float)idx);
    return make_uint2(pack_bf16x2(__fmul_rn(t, a ? V.v[4] : V.v[0]), __fmul_rn(t, a ? V.v[5] : V.v[1])),
                      pack_bf16x2(__fmul_rn(t, a ? V.v[6] : V.v[2]), __fmul_rn(t, a ? V.v[7] : V.v[3])));
  }
}

// The A operand of one row for one chunk of 64 weights (the 4 qs words of the
// chunk, cc = chunk index inside its 256-block): 32 registers of bf16 pairs.
// regs[8m + 2i] holds weights (16m + i, 16m + 4 + i) and regs[8m + 2i + 1]
// holds (16m + 8 + i, 16m + 12 + i) of the chunk, the slot order in which
// the token rows are transposed (the byte-permute lookup emits codes i,
// 4 + i, 8 + i, 12 + i of a word together).
template <int FMT>
__device__ __forceinline__ void decode_chunk(const BlkSc<FMT>& sc, int cc, const uint32_t (&qv)[4], const uint2* lut,
                                             const Values& V, uint32_t (&regs)[32]) {
#pragma unroll
  for (int m = 0; m < 4; m++) {
    const uint2 tw = table_words<FMT>(sc, cc, m, lut, V);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const Pair2 pr = lookup_slot(qv[m], i, tw.x, tw.y);
      regs[8 * m + 2 * i] = pr.lo;
      regs[8 * m + 2 * i + 1] = pr.hi;
    }
  }
}

__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t par, volatile uint32_t* abort_flag, int32_t* status) {
  for (uint32_t i = 0; i < (1u << 24); i++) {
    if (mbar_try_wait(bar, par)) return true;
    if ((i & 1023u) == 1023u && *abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(status, 2);
  return false;
}

// One producer warp's share of an (item, N tile): rows 32q .. 32q + 31 of its
// 128-row tile, all K chunks of 64. The decode of chunk c + 1 overlaps the
// tensor-memory store of chunk c: the store's completion is awaited (and the
// MMA warp signalled) only after the next chunk is in registers.
template <int FMT>
__device__ __forceinline__ bool pf_produce(const WDev& W, int64_t grow, int nch, int tile, int q, int r, int lane,
                                           const uint32_t* qbuf, uint64_t* qs_full, uint64_t* qs_empty,
                                           uint64_t* a_ready, uint64_t* a_free, uint32_t tmem, const uint2* lut,
                                           const Values& V, uint32_t& qi, uint32_t& ai, volatile uint32_t* abort_flag,
                                           int32_t* status) {
  const int nb = nch >> 2;
  BlkSc<FMT> sc = load_blk<FMT>(W, grow, 0);
  BlkSc<FMT> scn = nb > 1 ? load_blk<FMT>(W, grow, 1) : sc;  // the next 256-block, requested one block ahead
  const uint32_t tlane = tmem + ((uint32_t)(32 * q) << 16) + TM_A + (tile ? 32u : 0u);
  uint32_t ra[32], rb[32];
  int pend_sa = -1;  // stage of the chunk whose store is in flight
  // Decode chunk c into regs (registers only: the A stage is claimed after
  // the decode, just before the tensor-memory store, so the decode overlaps
  // the MMAs still reading that stage). Returns false after a failed wait.
  auto decode = [&](int c, uint32_t (&regs)[32]) -> bool {
    const int s = qi % PF_SQ;
    if ((c & 3) == 0) {
      if (c > 0) {
        sc = scn;
        if ((c >> 2) + 1 < nb) scn = load_blk<FMT>(W, grow, (c >> 2) + 1);
      }
      if (!pf_wait(&qs_full[s], (qi / PF_SQ) & 1, abort_flag, status)) return false;
    }
    // qs tiles arrive with the 64-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r >> 1) & 3)
    const uint4 qw = *reinterpret_cast<const uint4*>(qbuf + (size_t)s * (PF_Q_BYTES / 4) + (tile ? 128 * 16 : 0) +
                                                     r * 16 + 4 * ((c & 3) ^ ((r >> 1) & 3)));
    const uint32_t qv[4] = {qw.x, qw.y, qw.z, qw.w};
    decode_chunk<FMT>(sc, c & 3, qv, lut, V, regs);
    if ((c & 3) == 3) {  // the qs stage has been read in full
      __syncwarp();
      if (lane == 0) mbar_arrive(&qs_empty[s]);
      qi++;
    }
    return true;
  };
  // the next A stage, once the MMAs that read it last have completed; -1 after a failed wait
  auto claim = [&]() -> int {
    const int sa = ai % PF_SA;
    if (!pf_wait(&a_free[sa], ((ai / PF_SA) & 1) ^ 1, abort_flag, status)) return -1;
    ai++;
    return sa;
  };
  auto publish = [&]() {  // the pending chunk's store is complete: hand its stage to the MMA warp
    if (pend_sa < 0) return;
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&a_ready[pend_sa]);
  };
  for (int c = 0; c < nch; c += 2) {
    int sa;
    if (!decode(c, ra)) {
      tmem_wait_st();
      return false;
    }
    publish();
    if ((sa = claim()) < 0) {
      tmem_wait_st();
      return false;
    }
    tmem_st32(tlane + 64u * sa, ra);
    pend_sa = sa;
    if (!decode(c + 1, rb)) {
      tmem_wait_st();
      return false;
    }
    publish();
    if ((sa = claim()) < 0) {
      tmem_wait_st();
      return false;
    }
    tmem_st32(tlane + 64u * sa, rb);
    pend_sa = sa;
  }
  publish();
  return true;
}

template <int MODE, int F0, int F1>
__global__ void __launch_bounds__(PF_THREADS, 2) k_pf_gemm(const __grid_constant__ CUtensorMap q0,
                                                           const __grid_constant__ CUtensorMap q1,
                                                           const __grid_constant__ CUtensorMap bmap,
                                                           const __grid_constant__ PfArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* bbuf = smem;                                   // [SB][128 rows][128 B], 1024-aligned
  uint32_t* qbuf = reinterpret_cast<uint32_t*>(smem + PF_SB * PF_B_BYTES);  // [SQ][2][128][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PF_SB * PF_B_BYTES + PF_SQ * PF_Q_BYTES);
  uint64_t* qs_full = bars;
  uint64_t* qs_empty = qs_full + PF_SQ;
  uint64_t* b_full = qs_empty + PF_SQ;
  uint64_t* b_empty = b_full + PF_SB;
  uint64_t* a_ready = b_empty + PF_SB;
  uint64_t* a_free = a_ready + PF_SA;
  uint64_t* d_full = a_free + PF_SA;
  uint64_t* d_empty = d_full + 1;
  uint2* lut0 = reinterpret_cast<uint2*>(bars + PF_NBAR);
  uint2* lut1 = lut0 + 64;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(lut1 + 64);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  build_lut_pf<F0>(lut0, A.V);
  build_lut_pf<F1>(lut1, A.V);
  if (threadIdx.x == 0) {
    for (int s = 0; s < PF_SQ; s++) {
      mbar_init(&qs_full[s], 1);
      mbar_init(&qs_empty[s], 8);
    }
    for (int s = 0; s < PF_SB; s++) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < PF_SA; s++) {
      mbar_init(&a_ready[s], 8);
      mbar_init(&a_free[s], 1);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == PF_MMA_WARP) tmem_alloc(tmem_holder, TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int nitems = A.E * A.mtiles;
  const int nch = A.K / 64;

  if (warp == PF_TMA_WARP) {  // qs tiles, one 256-block ahead of the producers per stage
    if (lane == 0) {
      uint32_t qi = 0;
      for (int item = blockIdx.x; item < nitems && !*abort_flag; item += gridDim.x) {
        const int e = item / A.mtiles, mt = item % A.mtiles;
        const int ne = A.counts[e];
        int r0, r1;
        if (MODE == 0) {
          r0 = e * A.rows + 128 * mt;
          r1 = r0;
        } else {
          r0 = e * A.rows + 256 * mt;
          r1 = r0 + 128;
        }
        bool ok = true;
        for (int n0 = 0; n0 < ne && ok; n0 += PF_NMAX) {
          for (int c = 0; c < nch; c += 4) {
            const int s = qi % PF_SQ;
            if (!(ok = pf_wait(&qs_empty[s], ((qi / PF_SQ) & 1) ^ 1, abort_flag, A.status))) break;
            uint32_t* dst = qbuf + (size_t)s * (PF_Q_BYTES / 4);
            mbar_arrive_expect_tx(&qs_full[s], PF_Q_BYTES);
            tma_load_2d(dst, &q0, (c >> 2) * 16, r0, &qs_full[s]);
            tma_load_2d(dst + 128 * 16, &q1, (c >> 2) * 16, r1, &qs_full[s]);
            qi++;
          }
        }
      }
    }
  } else if (warp == PF_BTMA_WARP) {  // token rows of each K chunk
    if (lane == 0) {
      uint32_t bi = 0;
      for (int item = blockIdx.x; item < nitems && !*abort_flag; item += gridDim.x) {
        const int e = item / A.mtiles;
        const int ne = A.counts[e], off = A.offsets[e];
        bool ok = true;
        for (int n0 = 0; n0 < ne && ok; n0 += PF_NMAX) {
          const int npad = (((ne - n0) < PF_NMAX ? (ne - n0) : PF_NMAX) + 15) & ~15;
          for (int c = 0; c < nch; c++) {
            const int s = bi % PF_SB;
            if (!(ok = pf_wait(&b_empty[s], ((bi / PF_SB) & 1) ^ 1, abort_flag, A.status))) break;
            uint8_t* dst = bbuf + (size_t)s * PF_B_BYTES;
            mbar_arrive_expect_tx(&b_full[s], (uint32_t)npad * 128);
            for (int bx = 0; bx < npad / 16; bx++)
              tma_load_2d(dst + bx * 2048, &bmap, c * 64, off + n0 + 16 * bx, &b_full[s]);
            bi++;
          }
        }
      }
    }
  } else if (warp == PF_MMA_WARP) {
    if (lane == 0) {
      uint32_t ai = 0, bi = 0, di = 0;
      for (int item = blockIdx.x; item < nitems && !*abort_flag; item += gridDim.x) {
        const int e = item / A.mtiles;
        const int ne = A.counts[e];
        for (int n0 = 0; n0 < ne; n0 += PF_NMAX) {
          const int npad = (((ne - n0) < PF_NMAX ? (ne - n0) : PF_NMAX) + 15) & ~15;
          const uint32_t idesc = idesc_bf16_m128((uint32_t)npad);
          if (!pf_wait(d_empty, (di & 1) ^ 1, abort_flag, A.status)) break;
          tc_fence_after();
          for (int c = 0; c < nch; c++) {
            const int sa = ai % PF_SA, sb = bi % PF_SB;
            if (!pf_wait(&a_ready[sa], (ai / PF_SA) & 1, abort_flag, A.status)) break;
            if (!pf_wait(&b_full[sb], (bi / PF_SB) & 1, abort_flag, A.status)) break;
            tc_fence_after();
            const uint32_t bbase = smem_u32(bbuf + (size_t)sb * PF_B_BYTES);
            const uint32_t abase = tmem + TM_A + 64u * sa;
#pragma unroll
            for (int j = 0; j < 4; j++) {
              const uint64_t bd = sdesc_kmajor_sw128(bbase + 32u * j);
              const uint32_t acc = (c | j) != 0;
              mma_ts(tmem + TM_D0, abase + 8u * j, bd, idesc, acc);
              mma_ts(tmem + TM_D1, abase + 32u + 8u * j, bd, idesc, acc);
            }
            tc_commit(&a_free[sa]);
            tc_commit(&b_empty[sb]);
            ai++;
            bi++;
          }
          tc_commit(d_full);
          di++;
        }
      }
    }
  } else {
    // ---- producer warps 0..7: tile = warp / 4, lanes (32 q .. 32 q + 31) of tensor memory
    const int tile = warp >> 2, q = warp & 3, r = 32 * q + lane;
    const WDev& W = tile ? A.w1 : A.w0;
    const uint2* lut = tile ? lut1 : lut0;
    uint32_t qi = 0, ai = 0, di = 0;
    for (int item = blockIdx.x; item < nitems && !*abort_flag; item += gridDim.x) {
      const int e = item / A.mtiles, mt = item % A.mtiles;
      const int ne = A.counts[e], off = A.offsets[e];
      const int64_t grow = MODE == 0 ? (int64_t)e * A.rows + 128 * mt + r
                                     : (int64_t)e * A.rows + 256 * mt + 128 * tile + r;
      for (int n0 = 0; n0 < ne; n0 += PF_NMAX) {
        const int ncols = ((ne - n0) < PF_NMAX ? (ne - n0) : PF_NMAX);
        const int npad = (ncols + 15) & ~15;
        const bool ok = tile == 0
                            ? pf_produce<F0>(W, grow, nch, tile, q, r, lane, qbuf, qs_full, qs_empty, a_ready, a_free, tmem,
                                             lut, A.V, qi, ai, abort_flag, A.status)
                            : pf_produce<F1>(W, grow, nch, tile, q, r, lane, qbuf, qs_full, qs_empty, a_ready, a_free, tmem,
                                             lut, A.V, qi, ai, abort_flag, A.status);
        if (!ok) break;
        // ---- epilogue of this (item, N tile)
        if (!pf_wait(d_full, di & 1, abort_flag, A.status)) break;
        tc_fence_after();
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        if (MODE == 0) {
          const int f = 128 * mt + r;  // row of gate and up
          const int Fdim = A.rows;
          const float dg = F0 == FMT_KS ? __half2float(__ushort_as_half(__ldg(A.w0.dv + (int64_t)e * Fdim + f))) : 1.f;
          const float du = F1 == FMT_KS ? __half2float(__ushort_as_half(__ldg(A.w1.dv + (int64_t)e * Fdim + f))) : 1.f;
          const int half = npad / 2;
          const int cbeg = tile * half, cend = cbeg + half;
          for (int c0 = cbeg; c0 < cend; c0 += 8) {
            float g8[8], u8[8];
            tmem_ld8(lane_base + TM_D0 + c0, g8);
            tmem_ld8(lane_base + TM_D1 + c0, u8);
#pragma unroll
            for (int i = 0; i < 8; i++) {
              const int n = c0 + i;
              if (n < ncols) {
                const float gv = g8[i] * dg, uv = u8[i] * du;
                const float h = silu_f32(gv) * uv;
                A.hs[(size_t)(off + n0 + n) * Fdim + perm16(f)] = f32_to_bf16_bits(h);
              }
            }
          }
        } else {
          const int H = A.rows;
          const int o = 256 * mt + 128 * tile + r;
          const float dr = (tile ? F1 : F0) == FMT_KS ? __half2float(__ushort_as_half(__ldg(W.dv + grow))) : 1.f;
          for (int c0 = 0; c0 < npad; c0 += 8) {
            float v8[8];
            tmem_ld8(lane_base + (tile ? TM_D1 : TM_D0) + c0, v8);
#pragma unroll
            for (int i = 0; i < 8; i++) {
              const int n = c0 + i;
              if (n < ncols) A.outp[(size_t)(off + n0 + n) * H + o] = v8[i] * dr;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(d_empty);
        di++;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == PF_MMA_WARP) tmem_dealloc(tmem, TM_COLS);
}

// ------------------------------------------------ gather, combine, sizing

// Xs[i] = slot-transposed x[token of pair perm[i]]; inv[perm[i]] = i.
__global__ void __launch_bounds__(256) k_pf_gather(const uint16_t* __restrict__ x, int H, int topk,
                                                   const int32_t* __restrict__ perm, const int32_t* __restrict__ offsets,
                                                   int E, uint16_t* __restrict__ xs, int32_t* __restrict__ inv) {
  const int nvalid = offsets[E];
  const int groups = H / 16;
  const int64_t n = (int64_t)nvalid * groups;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n; g += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(g / groups), grp = (int)(g % groups);
    const int pair = perm[i];
    if (grp == 0) inv[pair] = i;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(pair / topk) * H + 16 * grp);
    const uint4 a = src[0], b = src[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[8];
    // out[4i + j] = in[i + 4j]: output word 2i = (in[i], in[i+4]), word 2i+1 = (in[i+8], in[i+12])
#pragma unroll
    for (int i2 = 0; i2 < 4; i2++) {
      const int wa = i2 >> 1;
      const uint32_t sel = (i2 & 1) ? 0x7632u : 0x5410u;
      o[2 * i2] = prmt(w[wa], w[wa + 2], sel);
      o[2 * i2 + 1] = prmt(w[wa + 4], w[wa + 6], sel);
    }
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)i * H + 16 * grp);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// y[t][o] = bf16(sum over slots j in order of p[t][j] * outp[inv[t*topk + j]][o])
// (inv == nullptr: row t*topk + j); float32 into yf instead when yf is set.
__global__ void __launch_bounds__(256) k_pf_combine(const float* __restrict__ outp, const int32_t* __restrict__ inv,
                                                    const float* __restrict__ p, int T, int topk, int H,
                                                    uint16_t* __restrict__ y, float* __restrict__ yf) {
  const int64_t n = (int64_t)T * (H / 4);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n; g += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(g / (H / 4)), o4 = (int)(g % (H / 4));
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < topk; j++) {
      const int pos = inv ? inv[t * topk + j] : t * topk + j;
      if (pos < 0) continue;
      const float pw = __ldg(p + t * topk + j);
      const float4 v = __ldg(reinterpret_cast<const float4*>(outp + (size_t)pos * H) + o4);
      s.x += pw * v.x;
      s.y += pw * v.y;
      s.z += pw * v.z;
      s.w += pw * v.w;
    }
    if (yf) {
      reinterpret_cast<float4*>(yf + (size_t)t * H)[o4] = s;
    } else {
      uint2 out;
      out.x = pack_bf16x2(s.x, s.y);
      out.y = pack_bf16x2(s.z, s.w);
      reinterpret_cast<uint2*>(y + (size_t)t * H)[o4] = out;
    }
  }
}

int launch_combine(const float* rows, const float* p, int T, int topk, int H, uint16_t* y, cudaStream_t st,
                   int num_sms) {
  const int64_t n = (int64_t)T * (H / 4);
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 16);
  k_pf_combine<<<std::max(blocks, 1), 256, 0, st>>>(rows, nullptr, p, T, topk, H, y, nullptr);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

PrefillWs prefill_ws(int T, int topk, int experts, int hidden, int inter) {
  PrefillWs ws = {};
  const int P = T * topk;
  ws.npairs = P;
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.counts = o;
  o = align256(o + (size_t)experts * 4);
  ws.offsets = o;
  o = align256(o + (size_t)(experts + 1) * 4);
  ws.perm = o;
  o = align256(o + (size_t)P * 4);
  ws.tiles = o;  // inverse permutation
  o = align256(o + (size_t)P * 4);
  ws.xs = o;  // route scratch, then the gathered rows
  o = align256(o + route_scratch_ints(P, experts) * 4);
  const size_t cc = ws.xs;
  ws.xs = o;
  o = align256(o + (size_t)P * hidden * 2);
  ws.hs = o;
  o = align256(o + (size_t)P * inter * 2);
  ws.outp = o;
  o = align256(o + (size_t)P * hidden * 4);
  ws.total = o;
  ws.max_tiles = (int)cc;  // offset of the route scratch
  return ws;
}

static int make_rows_map(CUtensorMap* map, const void* base, int rows, int cols) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return -4;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -4;
}

static int make_qs_tile_map(CUtensorMap* map, const WDev& w) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return -4;
  const cuuint64_t dims[2] = {(cuuint64_t)(w.cols / 16), (cuuint64_t)w.experts * (cuuint64_t)w.rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(w.cols / 16) * 4};
  const cuuint32_t box[2] = {16, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(w.qs), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -4;
}

template <int MODE, int F0, int F1>
static int launch_gemm(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb, const PfArgs& a,
                       cudaStream_t st, int num_sms) {
  auto kern = k_pf_gemm<MODE, F0, F1>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PF_SMEM) != cudaSuccess) return -4;
    attr = true;
  }
  const int grid = std::max(1, std::min(2 * num_sms, a.E * a.mtiles));
  kern<<<grid, PF_THREADS, PF_SMEM, st>>>(m0, m1, mb, a);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

template <int MODE>
static int dispatch_gemm(int f0, int f1, const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb,
                         const PfArgs& a, cudaStream_t st, int num_sms) {
  if (f0 == FMT_KS && f1 == FMT_KS) return launch_gemm<MODE, FMT_KS, FMT_KS>(m0, m1, mb, a, st, num_sms);
  if (f0 == FMT_KS && f1 == FMT_K) return launch_gemm<MODE, FMT_KS, FMT_K>(m0, m1, mb, a, st, num_sms);
  if (f0 == FMT_K && f1 == FMT_KS) return launch_gemm<MODE, FMT_K, FMT_KS>(m0, m1, mb, a, st, num_sms);
  return launch_gemm<MODE, FMT_K, FMT_K>(m0, m1, mb, a, st, num_sms);
}

int launch_moe_prefill(const WDev& g, int fg, const WDev& u, int fu, const WDev& d, int fd, const Values& V,
                       const uint16_t* x, int T, const int32_t* ids, const float* p, int topk, uint16_t* y, float* yf,
                       int ebase, char* ws, cudaStream_t st, int num_sms) {
  const int H = g.cols, F = g.rows, E = g.experts;
  const PrefillWs L = prefill_ws(T, topk, E, H, F);
  const int P = T * topk;
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + L.tiles);
  int32_t* cc = reinterpret_cast<int32_t*>(ws + (size_t)L.max_tiles);
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  uint16_t* hs = reinterpret_cast<uint16_t*>(ws + L.hs);
  float* outp = reinterpret_cast<float*>(ws + L.outp);

  if (cudaMemsetAsync(inv, 0xFF, (size_t)P * 4, st) != cudaSuccess) return -4;
  int rc = launch_route(ids, T, topk, E, counts, offsets, perm, status, cc, st, ebase, yf != nullptr);
  if (rc) return rc;
  {
    const int64_t n = (int64_t)P * (H / 16);
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 16);
    k_pf_gather<<<std::max(blocks, 1), 256, 0, st>>>(x, H, topk, perm, offsets, E, xs, inv);
  }
  CUtensorMap mg, mu, md, mx, mh;
  if (make_qs_tile_map(&mg, g) || make_qs_tile_map(&mu, u) || make_qs_tile_map(&md, d)) return -4;
  if (make_rows_map(&mx, xs, P, H) || make_rows_map(&mh, hs, P, F)) return -4;
  PfArgs a0 = {};
  a0.w0 = g;
  a0.w1 = u;
  a0.V = V;
  a0.counts = counts;
  a0.offsets = offsets;
  a0.perm = perm;
  a0.p = p;
  a0.hs = hs;
  a0.outp = outp;
  a0.status = status;
  a0.E = E;
  a0.K = H;
  a0.rows = F;
  a0.mtiles = F / 128;
  if ((rc = dispatch_gemm<0>(fg, fu, mg, mu, mx, a0, st, num_sms))) return rc;
  PfArgs a1 = a0;
  a1.w0 = d;
  a1.w1 = d;
  a1.K = F;
  a1.rows = H;
  a1.mtiles = H / 256;
  if ((rc = dispatch_gemm<1>(fd, fd, md, md, mh, a1, st, num_sms))) return rc;
  {
    const int64_t n = (int64_t)T * (H / 4);
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 16);
    k_pf_combine<<<std::max(blocks, 1), 256, 0, st>>>(outp, inv, p, T, topk, H, y, yf);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

// ------------------------------------------------ switch linear, GEMM form
// y[pair] = W_{ids[pair]} x[pair / topk] for many pairs: the same grouping,
// gather and down-mode grouped GEMM as the prefill, then the per-pair rows are
// put back in pair order (zero rows for out-of-range ids).

__global__ void __launch_bounds__(256) k_sw_scatter(const float* __restrict__ outp, const int32_t* __restrict__ inv,
                                                    int P, int rows, float* __restrict__ y) {
  const int64_t n = (int64_t)P * (rows / 4);
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n; g += (int64_t)gridDim.x * blockDim.x) {
    const int pair = (int)(g / (rows / 4)), o4 = (int)(g % (rows / 4));
    const int pos = inv[pair];
    const float4 v = pos >= 0 ? __ldg(reinterpret_cast<const float4*>(outp + (size_t)pos * rows) + o4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(y + (size_t)pair * rows)[o4] = v;
  }
}

namespace {
struct SwGemmWs {
  size_t status, counts, offsets, perm, inv, cc, xs, outp, total;
};
SwGemmWs sw_gemm_ws(int T, int topk, int experts, int rows, int cols) {
  SwGemmWs ws = {};
  const int P = T * topk;
  size_t o = 0;
  ws.status = o;
  o = align256(o + 16);
  ws.counts = o;
  o = align256(o + (size_t)experts * 4);
  ws.offsets = o;
  o = align256(o + (size_t)(experts + 1) * 4);
  ws.perm = o;
  o = align256(o + (size_t)P * 4);
  ws.inv = o;
  o = align256(o + (size_t)P * 4);
  ws.cc = o;
  o = align256(o + route_scratch_ints(P, experts) * 4);
  ws.xs = o;
  o = align256(o + (size_t)P * cols * 2);
  ws.outp = o;
  o = align256(o + (size_t)P * rows * 4);
  ws.total = o;
  return ws;
}
}  // namespace

size_t switch_gemm_ws(int T, int topk, int experts, int rows, int cols) {
  return sw_gemm_ws(T, topk, experts, rows, cols).total;
}

int launch_switch_gemm(const WDev& w, int fmt, const Values& V, const uint16_t* x, int T, const int32_t* ids,
                       int topk, float* y, char* ws, cudaStream_t st, int num_sms) {
  const int E = w.experts, K = w.cols, R = w.rows;
  const SwGemmWs L = sw_gemm_ws(T, topk, E, R, K);
  const int P = T * topk;
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
  int32_t* cc = reinterpret_cast<int32_t*>(ws + L.cc);
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + L.xs);
  float* outp = reinterpret_cast<float*>(ws + L.outp);
  if (cudaMemsetAsync(inv, 0xFF, (size_t)P * 4, st) != cudaSuccess) return -4;
  int rc = launch_route(ids, T, topk, E, counts, offsets, perm, status, cc, st);
  if (rc) return rc;
  {
    const int64_t n = (int64_t)P * (K / 16);
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 16);
    k_pf_gather<<<std::max(blocks, 1), 256, 0, st>>>(x, K, topk, perm, offsets, E, xs, inv);
  }
  CUtensorMap mw, mx;
  if (make_qs_tile_map(&mw, w) || make_rows_map(&mx, xs, P, K)) return -4;
  PfArgs a = {};
  a.w0 = w;
  a.w1 = w;
  a.V = V;
  a.counts = counts;
  a.offsets = offsets;
  a.perm = perm;
  a.outp = outp;
  a.status = status;
  a.E = E;
  a.K = K;
  a.rows = R;
  a.mtiles = R / 256;
  if ((rc = dispatch_gemm<1>(fmt, fmt, mw, mw, mx, a, st, num_sms))) return rc;
  {
    const int64_t n = (int64_t)P * (R / 4);
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 16);
    k_sw_scatter<<<std::max(blocks, 1), 256, 0, st>>>(outp, inv, P, R, y);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

// ------------------------------------------------------ A-operand inspection
// The producer's A operand of rows [row0, row0 + nrows) of expert e, every
// column, written to global memory in k order (out[r][k], bf16 bits): the
// same block scales, tables and chunk decode (decode_chunk) the producers of
// k_pf_gemm store into tensor memory, with the slot order undone. IQ2_K:
// bf16_rn((d * float(idx)) * value); IQ2_KS: bf16_rn(float(idx) * value), its
// row scale d being applied to the accumulator in the epilogue. One thread
// per row.
template <int FMT>
__global__ void __launch_bounds__(128) k_pf_a_tile(WDev w, int expert, int row0, int nrows, Values V,
                                                   uint16_t* __restrict__ out) {
  __shared__ uint2 lut[64];
  build_lut_pf<FMT>(lut, V);
  __syncthreads();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= nrows) return;
  const int64_t grow = (int64_t)expert * w.rows + row0 + r;
  const int wpr = w.cols / 16;
  BlkSc<FMT> sc = load_blk<FMT>(w, grow, 0);
  for (int c = 0; c < w.cols / 64; c++) {
    if ((c & 3) == 0) sc = load_blk<FMT>(w, grow, c >> 2);
    uint32_t qv[4];
    for (int m = 0; m < 4; m++) qv[m] = __ldg(w.qs + grow * wpr + 4 * c + m);
    uint32_t regs[32];
    decode_chunk<FMT>(sc, c & 3, qv, lut, V, regs);
    uint16_t* o = out + (size_t)r * w.cols + 64 * c;
    for (int m = 0; m < 4; m++)
      for (int i = 0; i < 4; i++) {
        const uint32_t lo = regs[8 * m + 2 * i], hi = regs[8 * m + 2 * i + 1];
        o[16 * m + i] = (uint16_t)(lo & 0xffffu);
        o[16 * m + 4 + i] = (uint16_t)(lo >> 16);
        o[16 * m + 8 + i] = (uint16_t)(hi & 0xffffu);
        o[16 * m + 12 + i] = (uint16_t)(hi >> 16);
      }
  }
}

int launch_pf_a_tile(const WDev& w, int fmt, int expert, int row0, int nrows, const Values& V, uint16_t* out,
                     cudaStream_t st) {
  const int blocks = (nrows + 127) / 128;
  if (fmt == FMT_KS) k_pf_a_tile<FMT_KS><<<blocks, 128, 0, st>>>(w, expert, row0, nrows, V, out);
  else k_pf_a_tile<FMT_K><<<blocks, 128, 0, st>>>(w, expert, row0, nrows, V, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
