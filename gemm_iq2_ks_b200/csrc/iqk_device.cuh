// Device-side building blocks shared by the IQ2_KS / IQ2_K kernels (sm_100a).
//
// Stream geometry follows the mlx-iqk 0.1.1 project page, section "Format"
// (IQ2_KS: 2-bit codes, 32-weight sub-blocks with a 5-bit signed scale index
// split over scl/sch, an alphabet bit, an fp16 row scale; IQ2_K: 16-weight
// sub-blocks with a 4-bit offset-8 index and an alphabet bit, fp16 scale per
// 256 weights). The bit packing inside scl/sch/sex is documented in iqk.h.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace iqk {

enum : int { FMT_KS = 0, FMT_K = 1 };

// Device view of one stacked weight tensor.
struct WDev {
  const uint32_t* qs;
  const uint32_t* scl;
  const uint8_t* sch;
  const void* sex;
  const uint16_t* dv;
  const uint8_t* slots;  // scale-slot images (iqk_pack_slots), or null
  int32_t experts, rows, cols;
};

struct Values {
  float v[8];
};

// Per-row element counts of each plane.
template <int FMT>
struct Geo {
  static __host__ __device__ __forceinline__ int64_t qs_w(int cols) { return cols / 16; }
  static __host__ __device__ __forceinline__ int64_t scl_w(int cols) { return FMT == FMT_KS ? cols / 256 : cols / 128; }
  static __host__ __device__ __forceinline__ int64_t sub_n(int cols) { return cols / 256; }  // sch / sex entries
  static __host__ __device__ __forceinline__ int64_t dv_n(int cols) { return FMT == FMT_KS ? 1 : cols / 256; }
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_4(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                           uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  mma_bf16_4(d[0], d[1], d[2], d[3], a0, a1, a2, a3, b0, b1);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase. Returns false if the bound expired.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t max_iters = (1u << 24)) {
  for (uint32_t i = 0; i < max_iters; i++) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  return false;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase, the bound in nanoseconds of the GPU's
// global timer. Returns false once `limit_ns` has passed without the phase
// completing.
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 >= limit_ns) return false;
  }
}

// Device-scope relaxed load (polling a counter another SM adds to), and the
// acquire fence that, after such a load has seen a writer's fence + add,
// orders this thread's later loads after the writer's earlier stores.
__device__ __forceinline__ int32_t ld_relaxed_s32(const int32_t* p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// Device-scope acquire load: once it reads a value a writer's fence + add
// produced, this thread's later loads see what the writer stored before.
__device__ __forceinline__ int32_t ld_acquire_s32(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bound of the waits that let a warp's copies still in flight land after one
// of its waits expired (the copies complete on their own; this only guards
// against a wedged copy engine).
constexpr uint64_t kDrainWaitNs = 2000000000ull;

// Fetch a TMA descriptor (a kernel parameter) ahead of its first use.
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled TMA load (no multicast) into shared memory, completion on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk copy (no multicast) of `bytes` from global into shared memory,
// completion on `bar`; both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// silu(g) = g / (1 + e^-g), evaluated as g * sigmoid(g) from e = exp(-|g|),
// which never overflows: sigmoid(g) = 1 / (1 + e) for g >= 0 and e / (1 + e)
// below. The plain quotient overflows e^-g to infinity below g = -88 and
// returns 0 where silu(g) is still a normal float (about -90 * e^-90).
__device__ __forceinline__ float silu_f32(float g) {
  const float e = expf(-fabsf(g));
  const float r = 1.0f / (1.0f + e);
  return g * (g >= 0.f ? r : e * r);
}

// bf16 helpers (bit patterns)
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------- code lookup
//
// The tensor-core operand for one qs word and one "slot" i (0..3): the bytes
// of u = (q >> 2i) & 0x03030303 hold the codes of weights i, i+4, i+8, i+12
// of the word. With a 4-entry table laid out as bf16 entry c at bytes
// (2c, 2c+1) of the pair {t0, t1}, the byte-permute selector of a code is
// 0x22*c + 0x10 (nibbles 2c, 2c+1); one multiply-add builds the selectors of
// four codes at once (the FMA pipe), and each permute yields two weights.
struct Pair2 {
  uint32_t lo, hi;  // bf16x2 (w_i, w_{i+4}) and (w_{i+8}, w_{i+12})
};

__device__ __forceinline__ Pair2 lookup_slot(uint32_t q, int i, uint32_t t0, uint32_t t1) {
  uint32_t u = (q >> (2 * i)) & 0x03030303u;
  uint32_t s = u * 0x22u + 0x10101010u;
  Pair2 r;
  r.lo = prmt(t0, t1, s);
  r.hi = prmt(t0, t1, s >> 16);
  return r;
}

// Same, with the high selector's 16-bit shift done as a multiply-high by
// `k65536` (= 65536, held in a register the compiler cannot fold), which runs
// on the FMA pipe instead of the integer-logic pipe the permutes use.
__device__ __forceinline__ Pair2 lookup_slot_mh(uint32_t q, int i, uint32_t t0, uint32_t t1, uint32_t k65536) {
  uint32_t u = (q >> (2 * i)) & 0x03030303u;
  uint32_t s = u * 0x22u + 0x10101010u;
  uint32_t sh;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(sh) : "r"(s), "r"(k65536));
  Pair2 r;
  r.lo = prmt(t0, t1, s);
  r.hi = prmt(t0, t1, sh);
  return r;
}

// Same, with the 2i-bit pre-shift of slot i also done as a multiply-high by
// `k_shift` (= 2^(32 - 2i), opaque): balances the integer-logic and FMA pipes.
__device__ __forceinline__ Pair2 lookup_slot_mh2(uint32_t q, uint32_t t0, uint32_t t1, uint32_t k65536,
                                                 uint32_t k_shift) {
  uint32_t qs;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(qs) : "r"(q), "r"(k_shift));
  uint32_t u = qs & 0x03030303u;
  uint32_t s = u * 0x22u + 0x10101010u;
  uint32_t sh;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(sh) : "r"(s), "r"(k65536));
  Pair2 r;
  r.lo = prmt(t0, t1, s);
  r.hi = prmt(t0, t1, sh);
  return r;
}

__device__ __forceinline__ uint32_t opaque_u32(uint32_t v) {
  uint32_t r;
  asm volatile("mov.u32 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// 16 bytes through L2 only (no L1 allocation): call inputs read before a
// kernel's dependency wait.
__device__ __forceinline__ uint4 ld_cg_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// 16 bytes by a plain global load: data a preceding kernel of the same call
// wrote, read after the dependency wait (the wait orders those writes first).
__device__ __forceinline__ uint4 ld_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Position of k within its 16-group after the slot transpose used by the
// activation operand: element k = 16w + i + 4j lives at 16w + 4i + j.
__host__ __device__ __forceinline__ int perm16(int k) {
  return (k & ~15) | ((k & 3) << 2) | ((k >> 2) & 3);
}

}  // namespace iqk
