// K0: bit-exact float32 reconstruction of one expert (and its bf16 rounding).
//
// mlx-iqk 0.1.1 PKG-INFO, section "Format": w = d * float(scale_index) *
// values[4*alphabet + code], every step float32, in that order. Both products
// use __fmul_rn (no contraction into an FMA); the library is built without
// fast-math, so subnormal products are kept and zeros carry the IEEE sign.
#include "iqk_device.cuh"
#include "iqk_internal.h"

namespace iqk {

// One thread per qs word (16 weights): one sub-block (IQ2_K) or half of one
// (IQ2_KS); output written with 16-byte stores.
//
// FLOOR: the same loads and the same stores with the decode deleted. The
// loaded words are folded into one integer, m = q ^ scl ^ sch ^ (sex << 8) ^
// (dv << 16), and output word k of the thread's 16 (8 for bf16) is m ^ k, so
// every loaded byte reaches the output and nothing can be elided.
template <int FMT, bool BF16, bool FLOOR>
__global__ void __launch_bounds__(256) k_dequant(WDev w, int expert, Values V, void* __restrict__ out) {
  const int cols = w.cols;
  const int wpr = cols / 16;  // qs words per row
  const int64_t nwords = (int64_t)w.rows * wpr;
  for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < nwords;
       gi += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = gi / wpr;
    const int wk = (int)(gi - r * wpr);
    const int64_t er = (int64_t)expert * w.rows + r;
    const uint32_t q = __ldg(w.qs + er * wpr + wk);
    uint32_t s, h, x, dvb;
    int idx, a;
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
      h = 0u;
      x = __ldg(reinterpret_cast<const uint16_t*>(w.sex) + er * (cols / 256) + (j >> 4));
      dvb = __ldg(w.dv + er * (cols / 256) + (wk >> 4));
      idx = (int)((s >> (4 * (j & 7))) & 15) - 8;
      a = (x >> (j & 15)) & 1;
    }
    if constexpr (FLOOR) {
      const uint32_t m = q ^ s ^ h ^ (x << 8) ^ (dvb << 16);
      uint32_t* o32 = static_cast<uint32_t*>(out);
      if (!BF16) {
        uint4* dst = reinterpret_cast<uint4*>(o32 + r * cols + 16 * wk);
#pragma unroll
        for (int v = 0; v < 4; v++) dst[v] = make_uint4(m ^ (4u * v), m ^ (4u * v + 1), m ^ (4u * v + 2), m ^ (4u * v + 3));
      } else {
        uint4* dst = reinterpret_cast<uint4*>(o32 + r * (cols / 2) + 8 * wk);
        dst[0] = make_uint4(m, m ^ 1u, m ^ 2u, m ^ 3u);
        dst[1] = make_uint4(m ^ 4u, m ^ 5u, m ^ 6u, m ^ 7u);
      }
      continue;
    }
    const float d = __half2float(__ushort_as_half((unsigned short)dvb));
    const float t = __fmul_rn(d, (float)idx);
    const float p0 = __fmul_rn(t, a ? V.v[4] : V.v[0]);
    const float p1 = __fmul_rn(t, a ? V.v[5] : V.v[1]);
    const float p2 = __fmul_rn(t, a ? V.v[6] : V.v[2]);
    const float p3 = __fmul_rn(t, a ? V.v[7] : V.v[3]);
    float o[16];
#pragma unroll
    for (int k = 0; k < 16; k++) {
      const uint32_t c = (q >> (2 * k)) & 3u;
      o[k] = (c & 2) ? ((c & 1) ? p3 : p2) : ((c & 1) ? p1 : p0);
    }
    if (!BF16) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + r * cols + 16 * wk);
#pragma unroll
      for (int v = 0; v < 4; v++) dst[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + r * cols + 16 * wk);
      uint32_t p[8];
#pragma unroll
      for (int v = 0; v < 8; v++) p[v] = pack_bf16x2(o[2 * v], o[2 * v + 1]);
      dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
      dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
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
  int64_t blocks = (nwords + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (floor) dequant_kernel<true>(fmt, bf16, blocks, threads, st, w, expert, V, out);
  else dequant_kernel<false>(fmt, bf16, blocks, threads, st, w, expert, V, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
