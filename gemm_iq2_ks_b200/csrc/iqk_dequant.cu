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
template <int FMT, bool BF16>
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
    int idx, a;
    float d;
    if (FMT == FMT_KS) {
      const int j = wk >> 1;  // 32-weight sub-block
      const int64_t sb = er * (cols / 256) + (j >> 3);
      const uint32_t s = __ldg(w.scl + sb);
      const uint32_t h = __ldg(w.sch + sb);
      const uint32_t x = __ldg(reinterpret_cast<const uint8_t*>(w.sex) + sb);
      const int lo = (s >> (4 * (j & 7))) & 15;
      const int hi = (h >> (j & 7)) & 1;
      idx = (lo | (hi << 4)) - 16;
      a = (x >> (j & 7)) & 1;
      d = __half2float(__ushort_as_half(__ldg(w.dv + er)));
    } else {
      const int j = wk;  // 16-weight sub-block
      const uint32_t s = __ldg(w.scl + er * (cols / 128) + (j >> 3));
      const uint32_t x = __ldg(reinterpret_cast<const uint16_t*>(w.sex) + er * (cols / 256) + (j >> 4));
      idx = (int)((s >> (4 * (j & 7))) & 15) - 8;
      a = (x >> (j & 15)) & 1;
      d = __half2float(__ushort_as_half(__ldg(w.dv + er * (cols / 256) + (wk >> 4))));
    }
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

int launch_dequant(const WDev& w, int fmt, int expert, const Values& V, void* out, bool bf16,
                   cudaStream_t st, int num_sms) {
  const int64_t nwords = (int64_t)w.rows * (w.cols / 16);
  const int threads = 256;
  int64_t blocks = (nwords + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (fmt == FMT_KS) {
    if (bf16) k_dequant<FMT_KS, true><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
    else k_dequant<FMT_KS, false><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
  } else {
    if (bf16) k_dequant<FMT_K, true><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
    else k_dequant<FMT_K, false><<<(unsigned)blocks, threads, 0, st>>>(w, expert, V, out);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
