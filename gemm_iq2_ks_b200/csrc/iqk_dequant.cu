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
template <int FMT, bool BF16, bool FLOOR>
__global__ void __launch_bounds__(256, 8) k_dequant(WDev w, int expert, Values V, void* __restrict__ out) {
  const int cols = w.cols;
  const int wpr = cols / 16;  // qs words per row
  const int64_t nwords = (int64_t)w.rows * wpr;
  const int64_t ntiles = (nwords + 31) / 32;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t tile = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; tile < ntiles; tile += nwarps) {
    const int64_t gw = tile * 32 + lane;
    uint32_t q = 0u, s = 0u, h = 0u, x = 0u, dvb = 0u;
    int idx = 0, a = 0;
    if (gw < nwords) {
      const int64_t r = gw / wpr;
      const int wk = (int)(gw - r * wpr);
      const int64_t er = (int64_t)expert * w.rows + r;
      q = __ldg(w.qs + er * wpr + wk);
      if (FMT == FMT_KS) {
        const int j = wk >> 1;  // 32-weight sub-block
        const int64_t sb = er * (cols / 256) + (j >> 3);
        s = __ldg(w.scl + sb);
        h = __ldg(w.sch + sb);
        x = __ldg(reinterpret_cast<const uint8_t*>(w.sex) + sb);
        dvb = __ldg(w.dv + er);
        const int lo = (s >> (4 * (j & 7))) & 15;
        const int hi = (h >> (j & 7)) & 1;
        idx = (lo | (hi << 4)) - 16;
        a = (x >> (j & 7)) & 1;
      } else {
        const int j = wk;  // 16-weight sub-block
        s = __ldg(w.scl + er * (cols / 128) + (j >> 3));
        x = __ldg(reinterpret_cast<const uint16_t*>(w.sex) + er * (cols / 256) + (j >> 4));
        dvb = __ldg(w.dv + er * (cols / 256) + (wk >> 4));
        idx = (int)((s >> (4 * (j & 7))) & 15) - 8;
        a = (x >> (j & 15)) & 1;
      }
    }
    constexpr int kChunks = BF16 ? 2 : 4;     // 16-byte chunks per qs word
    constexpr int kPer = 16 / kChunks;         // weights per chunk
    constexpr int kLanesPerWord = kChunks;     // lanes sharing one word in a store
    if constexpr (FLOOR) {
      const uint32_t m = q ^ s ^ h ^ (x << 8) ^ (dvb << 16);
      uint32_t* o32 = static_cast<uint32_t*>(out);
#pragma unroll
      for (int v = 0; v < kChunks; v++) {
        const int src = v * (32 / kLanesPerWord) + lane / kLanesPerWord;  // the word this lane's chunk belongs to
        const uint32_t mv = __shfl_sync(0xffffffffu, m, src);
        const int64_t word = tile * 32 + src;
        const uint32_t k0 = 4u * (uint32_t)(lane % kLanesPerWord);  // first output word of the chunk
        if (word < nwords)
          *reinterpret_cast<uint4*>(o32 + word * (BF16 ? 8 : 16) + k0) =
              make_uint4(mv ^ k0, mv ^ (k0 + 1u), mv ^ (k0 + 2u), mv ^ (k0 + 3u));
      }
      continue;
    }
    const float d = __half2float(__ushort_as_half((unsigned short)dvb));
    const float t = __fmul_rn(d, (float)idx);
#pragma unroll
    for (int v = 0; v < kChunks; v++) {
      const int src = v * (32 / kLanesPerWord) + lane / kLanesPerWord;
      const uint32_t qv = __shfl_sync(0xffffffffu, q, src);
      const float tv = __shfl_sync(0xffffffffu, t, src);
      const int av = __shfl_sync(0xffffffffu, a, src);
      const int64_t word = tile * 32 + src;
      const float p0 = __fmul_rn(tv, av ? V.v[4] : V.v[0]);
      const float p1 = __fmul_rn(tv, av ? V.v[5] : V.v[1]);
      const float p2 = __fmul_rn(tv, av ? V.v[6] : V.v[2]);
      const float p3 = __fmul_rn(tv, av ? V.v[7] : V.v[3]);
      const int w0 = kPer * (lane % kLanesPerWord);  // first weight of the chunk within the word
      float o[kPer];
#pragma unroll
      for (int k = 0; k < kPer; k++) {
        const uint32_t c = (qv >> (2 * (w0 + k))) & 3u;
        o[k] = (c & 2) ? ((c & 1) ? p3 : p2) : ((c & 1) ? p1 : p0);
      }
      if (word >= nwords) continue;
      if (!BF16) {
        *reinterpret_cast<float4*>(static_cast<float*>(out) + word * 16 + w0) = make_float4(o[0], o[1], o[2], o[3]);
      } else {
        uint32_t pk[4];
#pragma unroll
        for (int k = 0; k < 4; k++) pk[k] = pack_bf16x2(o[2 * k], o[2 * k + 1]);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + word * 16 + w0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
}

template <bool FLOOR>
static void dequant_kernel(int fmt, bool bf16, int64_t blocks, int threads, cudaStream_t st, const WDev& w,
                           int expert, const Values& V, void* out) {
  if (fmt == FMT_KS) {
    if (bf16) k_dequant<FMT_KS, true, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
    else k_dequant<FMT_KS, false, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
  } else {
    if (bf16) k_dequant<FMT_K, true, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
    else k_dequant<FMT_K, false, FLOOR><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
  }
}

int launch_dequant(const WDev& w, int fmt, int expert, const Values& V, void* out, bool bf16, bool floor,
                   cudaStream_t st, int num_sms) {
  const int64_t nwords = (int64_t)w.rows * (w.cols / 16);
  const int threads = 256;
  // 32-word tiles, one per warp at a time; every warp gets the same number of
  // tiles (up to the last), with at most 8 resident blocks per SM
  const int64_t ntiles = (nwords + 31) / 32;
  const int64_t cap_warps = (int64_t)num_sms * 8 * (threads / 32);
  const int64_t per_warp = (ntiles + cap_warps - 1) / cap_warps;
  int64_t blocks = (ntiles + per_warp * (threads / 32) - 1) / (per_warp * (threads / 32));
  if (blocks < 1) blocks = 1;
  if (floor) dequant_kernel<true>(fmt, bf16, blocks, threads, st, w, expert, V, out);
  else dequant_kernel<false>(fmt, bf16, blocks, threads, st, w, expert, V, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
