// K0: bit-exact float32 reconstruction of one expert (and its bf16 rounding).
//
// mlx-iqk 0.1.1 PKG-INFO, section "Format": w = d * float(scale_index) *
// values[4*alphabet + code], every step float32, in that order. Both products
// use __fmul_rn (no contraction into an FMA); the library is built without
// fast-math, so subnormal products are kept and zeros carry the IEEE sign.
#include "iqk_device.cuh"
#include "iqk_internal.h"

namespace iqk {

// A warp takes 32 consecutive qs words (512 weights) at a time. Lane i loads
// word i and its scale fields (one sub-block for IQ2_K, half of one for
// IQ2_KS) and forms its factors; the words' outputs are contiguous (word gw
// owns elements [16 gw, 16 gw + 16) of the expert's row-major matrix), so the
// warp writes them with 16-byte stores of which each instruction covers 512
// consecutive bytes: store v, lane i writes 16-byte chunk 32 v + i, the
// factors of its word fetched from the owning lane by shuffles.
//
// FLOOR: the same loads and the same stores with the decode deleted. The
// loaded words are folded into one integer, m = q ^ scl ^ sch ^ (sex << 8) ^
// (dv << 16), and output word k of a qs word's 16 (8 for bf16) is m ^ k, so
// every loaded byte reaches the output and nothing can be elided.
// The loads of one qs word: the word and its scale fields.
struct DqLoads {
  uint32_t q, s, h, x, dvb;
};

// Row and word-in-row of word gw (rows of wpr words): a multiply-shift
// division while the expert's words fit 31 bits, else a 64-bit division.
__device__ __forceinline__ void dq_split(int64_t gw, int64_t nwords, int wpr, FastDiv fd, int64_t& r, int& wk) {
  if (nwords < (int64_t(1) << 31)) {
    const uint32_t r32 = fd.div((uint32_t)gw);
    r = r32;
    wk = (int)((uint32_t)gw - r32 * (uint32_t)wpr);
  } else {
    r = gw / wpr;
    wk = (int)(gw - r * wpr);
  }
}

template <int FMT>
__device__ __forceinline__ DqLoads dq_load(const WDev& w, int expert, int64_t gw, int64_t nwords, int wpr, FastDiv fd) {
  DqLoads L = {0u, 0u, 0u, 0u, 0u};
  if (gw >= nwords) return L;
  int64_t r;
  int wk;
  dq_split(gw, nwords, wpr, fd, r, wk);
  const int64_t er = (int64_t)expert * w.rows + r;
  L.q = __ldg(w.qs + er * wpr + wk);
  if (FMT == FMT_KS) {
    const int64_t sb = er * (w.cols / 256) + (wk >> 4);
    L.s = __ldg(w.scl + sb);
    L.h = __ldg(w.sch + sb);
    L.x = __ldg(reinterpret_cast<const uint8_t*>(w.sex) + sb);
    L.dvb = __ldg(w.dv + er);
  } else {
    L.s = __ldg(w.scl + er * (w.cols / 128) + (wk >> 3));
    L.x = __ldg(reinterpret_cast<const uint16_t*>(w.sex) + er * (w.cols / 256) + (wk >> 4));
    L.dvb = __ldg(w.dv + er * (w.cols / 256) + (wk >> 4));
  }
  return L;
}

template <int FMT, bool BF16, bool FLOOR>
__global__ void __launch_bounds__(256, 6) k_dequant(WDev w, int expert, Values V, FastDiv fd, void* __restrict__ out) {
  const int wpr = w.cols / 16;  // qs words per row
  const int64_t nwords = (int64_t)w.rows * wpr;
  const int64_t ntiles = (nwords + 31) / 32;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  constexpr int kChunks = BF16 ? 2 : 4;  // 16-byte chunks per qs word
  constexpr int kPer = 16 / kChunks;     // weights per chunk
  int64_t tile = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  // the next tile's loads are issued before this tile is decoded and stored
  DqLoads cur = tile < ntiles ? dq_load<FMT>(w, expert, tile * 32 + lane, nwords, wpr, fd) : DqLoads{0u, 0u, 0u, 0u, 0u};
  for (; tile < ntiles; tile += nwarps) {
    const DqLoads nxt = tile + nwarps < ntiles ? dq_load<FMT>(w, expert, (tile + nwarps) * 32 + lane, nwords, wpr, fd)
                                               : DqLoads{0u, 0u, 0u, 0u, 0u};
    int64_t r_unused;
    int wk;
    dq_split(tile * 32 + lane, nwords, wpr, fd, r_unused, wk);
    if constexpr (FLOOR) {
      const uint32_t m = cur.q ^ cur.s ^ cur.h ^ (cur.x << 8) ^ (cur.dvb << 16);
      uint32_t* o32 = static_cast<uint32_t*>(out);
#pragma unroll
      for (int v = 0; v < kChunks; v++) {
        const int src = v * (32 / kChunks) + lane / kChunks;  // the word this lane's chunk belongs to
        const uint32_t mv = __shfl_sync(0xffffffffu, m, src);
        const int64_t word = tile * 32 + src;
        const uint32_t k0 = 4u * (uint32_t)(lane % kChunks);  // first output word of the chunk
        if (word < nwords)
          *reinterpret_cast<uint4*>(o32 + word * (BF16 ? 8 : 16) + k0) =
              make_uint4(mv ^ k0, mv ^ (k0 + 1u), mv ^ (k0 + 2u), mv ^ (k0 + 3u));
      }
    } else {
      // this lane's word: its four reconstructed values d * idx * values[4a + c]
      int idx, a;
      if (FMT == FMT_KS) {
        const int j = wk >> 1;  // 32-weight sub-block
        const int lo = (cur.s >> (4 * (j & 7))) & 15;
        const int hi = (cur.h >> (j & 7)) & 1;
        idx = (lo | (hi << 4)) - 16;
        a = (cur.x >> (j & 7)) & 1;
      } else {
        const int j = wk;  // 16-weight sub-block
        idx = (int)((cur.s >> (4 * (j & 7))) & 15) - 8;
        a = (cur.x >> (j & 15)) & 1;
      }
      const float d = __half2float(__ushort_as_half((unsigned short)cur.dvb));
      const float t = __fmul_rn(d, (float)idx);
      const float p0 = __fmul_rn(t, a ? V.v[4] : V.v[0]);
      const float p1 = __fmul_rn(t, a ? V.v[5] : V.v[1]);
      const float p2 = __fmul_rn(t, a ? V.v[6] : V.v[2]);
      const float p3 = __fmul_rn(t, a ? V.v[7] : V.v[3]);
#pragma unroll
      for (int v = 0; v < kChunks; v++) {
        const int src = v * (32 / kChunks) + lane / kChunks;
        const int w0 = kPer * (lane % kChunks);  // first weight of the chunk within the word
        const uint32_t qv = __shfl_sync(0xffffffffu, cur.q, src) >> (2 * w0);
        const float v0 = __shfl_sync(0xffffffffu, p0, src), v1 = __shfl_sync(0xffffffffu, p1, src);
        const float v2 = __shfl_sync(0xffffffffu, p2, src), v3 = __shfl_sync(0xffffffffu, p3, src);
        const int64_t word = tile * 32 + src;
        float o[kPer];
#pragma unroll
        for (int k = 0; k < kPer; k++) {
          const uint32_t c = (qv >> (2 * k)) & 3u;
          o[k] = (c & 2) ? ((c & 1) ? v3 : v2) : ((c & 1) ? v1 : v0);
        }
        if (word >= nwords) continue;
        if (!BF16) {
          *reinterpret_cast<float4*>(static_cast<float*>(out) + word * 16 + w0) = make_float4(o[0], o[1], o[2], o[3]);
        } else {
          uint32_t pk[4];
#pragma unroll
          for (int k = 0; k < 4; k++) pk[k] = pack_bf16x2(o[2 * k], o[2 * k + 1]);
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + word * 16 + w0) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    cur = nxt;
  }
}

template <bool FLOOR>
static void dequant_kernel(int fmt, bool bf16, int64_t blocks, int threads, cudaStream_t st, const WDev& w,
                           int expert, const Values& V, void* out) {
  const FastDiv fd = FastDiv::of((uint32_t)(w.cols / 16));
  if (fmt == FMT_KS) {
    if (bf16) k_dequant<FMT_KS, true, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, fd, out);
    else k_dequant<FMT_KS, false, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, fd, out);
  } else {
    if (bf16) k_dequant<FMT_K, true, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, fd, out);
    else k_dequant<FMT_K, false, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, fd, out);
  }
}

int launch_dequant(const WDev& w, int fmt, int expert, const Values& V, void* out, bool bf16, bool floor,
                   cudaStream_t st, int num_sms) {
  const int64_t nwords = (int64_t)w.rows * (w.cols / 16);
  const int threads = 256;
  // 32-word tiles, one per warp at a time; every warp gets the same number of
  // tiles (up to the last), with at most 6 resident blocks per SM
  const int64_t ntiles = (nwords + 31) / 32;
  const int64_t cap_warps = (int64_t)num_sms * 6 * (threads / 32);
  const int64_t per_warp = (ntiles + cap_warps - 1) / cap_warps;
  int64_t blocks = (ntiles + per_warp * (threads / 32) - 1) / (per_warp * (threads / 32));
  if (blocks < 1) blocks = 1;
  if (floor) dequant_kernel<true>(fmt, bf16, blocks, threads, st, w, expert, V, out);
  else dequant_kernel<false>(fmt, bf16, blocks, threads, st, w, expert, V, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
