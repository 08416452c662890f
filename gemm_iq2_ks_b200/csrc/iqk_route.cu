// Prefill grouping: expert histogram, exclusive prefix sum and the stable
// permutation of (token, slot) pairs in expert order.
//
// mlx-iqk 0.1.1 PKG-INFO, section "Surface": the prefill path honours the
// caller's sort so "each expert's weights are read once per sorted prefill".
// Ties keep pair order, so the permutation is unique and deterministic.
#include "iqk_device.cuh"
#include "iqk_internal.h"

namespace iqk {

constexpr int kRouteChunk = 1024;  // pairs per CTA
constexpr int kRouteThreads = 256;

// counts[e] (atomics; order-free) and per-chunk histograms cc[chunk][e].
// An expert-parallel shard (ebase > 0 or silent) groups only the pairs whose
// id lies in its window [ebase, ebase + E), as ids - ebase, and skips the
// others without flagging them.
__global__ void __launch_bounds__(kRouteThreads) k_route_count(const int32_t* __restrict__ ids, int npairs, int E,
                                                               int ebase, int silent, int32_t* __restrict__ counts,
                                                               int32_t* __restrict__ cc, int32_t* __restrict__ status) {
  extern __shared__ int32_t hist[];  // [E]
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kRouteChunk;
  for (int i = threadIdx.x; i < kRouteChunk; i += blockDim.x) {
    const int p = base + i;
    if (p >= npairs) break;
    const int e = ids[p] - ebase;
    if (e < 0 || e >= E) {
      if (!silent) atomicOr(status, 1);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int h = hist[e];
    cc[(size_t)blockIdx.x * E + e] = h;
    if (h) atomicAdd(&counts[e], h);
  }
}

// offsets = exclusive scan of counts; cc[chunk][e] becomes the chunk's base.
__global__ void __launch_bounds__(1024) k_route_scan(int E, int nchunks, const int32_t* __restrict__ counts,
                                                     int32_t* __restrict__ offsets, int32_t* __restrict__ cc) {
  __shared__ int32_t part[1024];
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int s = 0;
  for (int e = e0; e < e0 + per && e < E; e++) s += counts[e];
  part[threadIdx.x] = s;
  __syncthreads();
  // Hillis-Steele inclusive scan over the per-thread sums
  for (int d = 1; d < (int)blockDim.x; d <<= 1) {
    const int v = threadIdx.x >= (unsigned)d ? part[threadIdx.x - d] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = part[threadIdx.x] - s;  // exclusive
  for (int e = e0; e < e0 + per && e < E; e++) {
    offsets[e] = run;
    int b = run;
    for (int c = 0; c < nchunks; c++) {
      const int h = cc[(size_t)c * E + e];
      cc[(size_t)c * E + e] = b;
      b += h;
    }
    run += counts[e];
  }
  if (threadIdx.x == blockDim.x - 1) offsets[E] = part[threadIdx.x];
}

// perm[base[chunk][e] + stable rank within the chunk] = pair.
__global__ void __launch_bounds__(kRouteThreads) k_route_scatter(const int32_t* __restrict__ ids, int npairs, int E,
                                                                 int ebase, const int32_t* __restrict__ cc,
                                                                 int32_t* __restrict__ perm) {
  extern __shared__ int32_t run[];  // [E] next free position per expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = cc[(size_t)blockIdx.x * E + e];
  __syncthreads();
  const int base = blockIdx.x * kRouteChunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  // 32-pair groups in pair order; warps take turns so ranks follow pair order
  for (int grp = 0; grp < kRouteChunk / 32; grp++) {
    if (grp % nwarps == warp) {
      const int p = base + grp * 32 + lane;
      const bool in = p < npairs;
      const int e = in ? ids[p] - ebase : -1;
      const bool valid = in && e >= 0 && e < E;
      const unsigned vmask = __ballot_sync(0xffffffffu, valid);
      const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1) & vmask;
      if (valid) {
        const int below = __popc(same & ((1u << lane) - 1u));
        perm[run[e] + below] = p;
      }
      __syncwarp();
      const int leader = same ? __ffs(same) - 1 : -1;
      if (valid && lane == leader) run[e] += __popc(same);
    }
    __syncthreads();
  }
}

// The same placement in two barriers when 32 x E counters fit shared memory:
// every 32-pair group (in pair order) counts its pairs per expert (match_any),
// one thread per expert turns the counts into each group's base (the chunk's
// base plus the counts of the groups before it), then every pair lands at its
// group's base plus its rank among the group's earlier pairs of its expert.
__global__ void __launch_bounds__(kRouteThreads) k_route_place(const int32_t* __restrict__ ids, int npairs, int E,
                                                               int ebase, const int32_t* __restrict__ cc,
                                                               int32_t* __restrict__ perm) {
  constexpr int G = kRouteChunk / 32;  // groups per chunk
  extern __shared__ int32_t gcnt[];    // [G][E]: counts, then bases
  for (int i = threadIdx.x; i < G * E; i += blockDim.x) gcnt[i] = 0;
  __syncthreads();
  const int base = blockIdx.x * kRouteChunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  int e_of[G / 8], below_of[G / 8];
  for (int k = 0; k < G / nwarps; k++) {
    const int grp = warp + k * nwarps;
    const int p = base + grp * 32 + lane;
    const bool in = p < npairs;
    const int e = in ? __ldg(ids + p) - ebase : -1;
    const bool valid = in && e >= 0 && e < E;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1) & vmask;
    e_of[k] = valid ? e : -1;
    below_of[k] = __popc(same & ((1u << lane) - 1u));
    if (valid && below_of[k] == 0) gcnt[grp * E + e] = __popc(same);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int b = cc[(size_t)blockIdx.x * E + e];
    for (int grp = 0; grp < G; grp++) {
      const int c = gcnt[grp * E + e];
      gcnt[grp * E + e] = b;
      b += c;
    }
  }
  __syncthreads();
  for (int k = 0; k < G / nwarps; k++) {
    const int grp = warp + k * nwarps;
    if (e_of[k] >= 0) perm[gcnt[grp * E + e_of[k]] + below_of[k]] = base + grp * 32 + lane;
  }
}

int launch_route(const int32_t* ids, int T, int topk, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* status, int32_t* cc, cudaStream_t st, int ebase, bool silent) {
  const int npairs = T * topk;
  const int nchunks = (npairs + kRouteChunk - 1) / kRouteChunk;
  const size_t hsm = (size_t)E * 4;
  if (hsm > 200 * 1024) return -3;
  if (cudaMemsetAsync(counts, 0, (size_t)E * 4, st) != cudaSuccess) return -4;
  if (cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return -4;
  if (hsm > 48 * 1024) {
    cudaFuncSetAttribute(k_route_count, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsm);
    cudaFuncSetAttribute(k_route_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsm);
  }
  k_route_count<<<nchunks, kRouteThreads, hsm, st>>>(ids, npairs, E, ebase, silent ? 1 : 0, counts, cc, status);
  k_route_scan<<<1, 1024, 0, st>>>(E, nchunks, counts, offsets, cc);
  const size_t gsm = (size_t)(kRouteChunk / 32) * E * 4;
  if (gsm <= 160 * 1024) {
    static size_t place_attr = 48 * 1024;
    if (gsm > place_attr) {
      if (cudaFuncSetAttribute(k_route_place, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsm) != cudaSuccess)
        return -4;
      place_attr = gsm;
    }
    k_route_place<<<nchunks, kRouteThreads, gsm, st>>>(ids, npairs, E, ebase, cc, perm);
  } else {
    k_route_scatter<<<nchunks, kRouteThreads, hsm, st>>>(ids, npairs, E, ebase, cc, perm);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace iqk
