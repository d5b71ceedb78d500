// build_tables.cu — Block-Union KV selection on the GPU.
//
// "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection", Abstract: the 2D block-sparse masks are turned into GQA-aware
// per-group KV block tables by a Q-block union and an intra-group union, the
// minimal tables that keep every selected block.
//
// The rows of one group (G heads x nQblk Q-blocks) are contiguous in the mask,
// so the union is an OR-reduction of an [G*nQblk, nKblk] byte matrix down its
// rows, and the table is the ordered list of nonzero columns.  One thread
// block cluster (up to 8 CTAs) owns one (mask, group): each CTA reduces a
// column slab with 16-, 4- or 1-byte loads, turns it into a bit set in shared
// memory, and compacts it with per-word popcounts and a block scan; each CTA
// stores its slab count into the shared memory of every CTA of its cluster
// (one cluster barrier), then places its entries.  No global scratch, no
// atomics on global memory, and the output is deterministic.  HBM-bound:
// every mask byte is read exactly once.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace ca {

#ifndef CA_BUILD_CTAS_PER_SM
#define CA_BUILD_CTAS_PER_SM 2
#endif
#ifndef CA_BUILD_UNROLL
#define CA_BUILD_UNROLL 8
#endif
#ifndef CA_BUILD_MIN_BLOCKS
#define CA_BUILD_MIN_BLOCKS 4
#endif
constexpr int kBuildThreads = 256;
constexpr int kRowUnroll = CA_BUILD_UNROLL;
constexpr int kMaxSlab = 8192;  // columns per CTA -> 256 bit-set words, one per thread

// Streaming (evict-first) loads: each mask byte is read exactly once.
__device__ __forceinline__ uint4 ldcs(const uint4* p) { return __ldcs(p); }
__device__ __forceinline__ uint32_t ldcs(const uint32_t* p) { return __ldcs(p); }
__device__ __forceinline__ uint8_t ldcs(const uint8_t* p) {
  return (uint8_t)__ldcs(reinterpret_cast<const unsigned char*>(p));
}

template <int VEC>
struct VecLoad;
template <>
struct VecLoad<16> {
  using T = uint4;
  __device__ static uint4 zero() { return make_uint4(0, 0, 0, 0); }
  __device__ static void orin(uint4& a, const uint4& b) {
    a.x |= b.x; a.y |= b.y; a.z |= b.z; a.w |= b.w;
  }
  // byte i of the 16 -> bit i
  __device__ static uint32_t bits(const uint4& a) {
    auto nb = [](uint32_t x) {
      uint32_t m = __vcmpne4(x, 0u);  // 0xFF in each nonzero byte
      return ((m >> 7) & 1u) | ((m >> 14) & 2u) | ((m >> 21) & 4u) | ((m >> 28) & 8u);
    };
    return nb(a.x) | (nb(a.y) << 4) | (nb(a.z) << 8) | (nb(a.w) << 12);
  }
};
template <>
struct VecLoad<4> {
  using T = uint32_t;
  __device__ static uint32_t zero() { return 0u; }
  __device__ static void orin(uint32_t& a, const uint32_t& b) { a |= b; }
  __device__ static uint32_t bits(const uint32_t& a) {
    uint32_t m = __vcmpne4(a, 0u);
    return ((m >> 7) & 1u) | ((m >> 14) & 2u) | ((m >> 21) & 4u) | ((m >> 28) & 8u);
  }
};
template <>
struct VecLoad<1> {
  using T = uint8_t;
  __device__ static uint8_t zero() { return 0; }
  __device__ static void orin(uint8_t& a, const uint8_t& b) { a |= b; }
  __device__ static uint32_t bits(const uint8_t& a) { return a != 0; }
};

// grid = (C, Hkv, nb), cluster = (C, 1, 1); slab = columns per CTA (multiple of 32).
template <int VEC>
__global__ void __launch_bounds__(kBuildThreads, CA_BUILD_MIN_BLOCKS)
    build_tables_kernel(const uint8_t* __restrict__ mask, int Hq, int Hkv, int nQblk, int nKblk,
                        int slab, int32_t* __restrict__ tables, int32_t* __restrict__ counts) {
  using V = VecLoad<VEC>;
  using T = typename V::T;
  __shared__ uint32_t bits[kMaxSlab / 32];
  __shared__ int word_off[kMaxSlab / 32];  // entries of the slab before word w
  __shared__ int warp_sum[kBuildThreads / 32];
  __shared__ int slab_count[8];  // [r]: set columns in the slab of cluster rank r

  // Phase 0 of the cluster barrier: this CTA is running.  Its wait (after the
  // loads) guarantees that every CTA of the cluster has started before any
  // CTA stores into another's shared memory.
  cluster_arrive_relaxed();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int C = (int)cluster.num_blocks();
  const int tid = threadIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int G = Hq / Hkv;
  const int R = G * nQblk;  // rows of this group

  const uint8_t* base = mask + ((size_t)b * Hq + (size_t)g * G) * (size_t)nQblk * nKblk;
  const int c0 = rank * slab;
  const int c1 = min(nKblk, c0 + slab);
  const int ncols = max(0, c1 - c0);
  const int nwords = (ncols + 31) >> 5;

  for (int w = tid; w < kMaxSlab / 32; w += kBuildThreads) bits[w] = 0u;
  __syncthreads();

  // ---- Q-block union + intra-group union: OR down the group's rows.
  const int ncv = ncols / VEC;  // nKblk % VEC == 0 and c0 % VEC == 0
  int CW = 1;
  while (CW < ncv && CW < kBuildThreads) CW <<= 1;
  const int RT = kBuildThreads / CW;
  const int rt = tid / CW;
  for (int v = tid % CW; v < ncv; v += CW) {
    T acc = V::zero();
    if (rt < R) {
      const T* p = reinterpret_cast<const T*>(base + (size_t)rt * nKblk + c0) + v;
      const size_t step = (size_t)RT * nKblk / VEC;
      int r = rt;
#pragma unroll kRowUnroll
      for (; r < R; r += RT) {
        V::orin(acc, ldcs(p));  // read once: stream past L2
        p += step;
      }
    }
    uint32_t m = V::bits(acc);
    if (m) {
      const int col = v * VEC;  // within slab
      atomicOr(&bits[col >> 5], m << (col & 31));
    }
  }
  __syncthreads();

  // ---- compaction: popcount per 32-column word, exclusive block scan.
  const int lane = tid & 31, warp = tid >> 5;
  uint32_t word = (tid < nwords) ? bits[tid] : 0u;
  int cnt = __popc(word);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int wbase = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kBuildThreads / 32; ++w) {
    wbase += (w < warp) ? warp_sum[w] : 0;
    tot += warp_sum[w];
  }
  if (tid < nwords) word_off[tid] = wbase + incl - cnt;

  // ---- cluster: every CTA learns every slab count.  Rank r's count goes to
  // slab_count[r] of each CTA; after the barrier all reads are local, so no
  // CTA touches another's shared memory once it may have exited.
  cluster_wait_acquire();
  if (tid < C) st_cluster_s32(mapa_rank(smem_u32(&slab_count[rank]), (uint32_t)tid), tot);
  cluster_arrive_release();
  cluster_wait_acquire();
  int before = 0, total = 0;
  for (int r = 0; r < C; ++r) {
    const int t = slab_count[r];
    before += (r < rank) ? t : 0;
    total += t;
  }

  int32_t* trow = tables + ((size_t)b * Hkv + g) * nKblk;
  // Word w is written by warp w % 8: lane l handles column 32w + l, at the
  // word's offset plus the set bits below l.
  for (int w = warp; w < nwords; w += kBuildThreads / 32) {
    const uint32_t x = bits[w];
    if ((x >> lane) & 1u)
      trow[before + word_off[w] + __popc(x & ((1u << lane) - 1u))] = c0 + w * 32 + lane;
  }
  // -1 padding of the positions [total, nKblk) that fall inside this slab.
  for (int p = max(total, c0) + tid; p < c1; p += kBuildThreads) trow[p] = -1;
  if (rank == 0 && tid == 0) counts[(size_t)b * Hkv + g] = total;
}

template __global__ void build_tables_kernel<16>(const uint8_t*, int, int, int, int, int,
                                                 int32_t*, int32_t*);
template __global__ void build_tables_kernel<4>(const uint8_t*, int, int, int, int, int, int32_t*,
                                                int32_t*);
template __global__ void build_tables_kernel<1>(const uint8_t*, int, int, int, int, int, int32_t*,
                                                int32_t*);

// Host launcher: picks the vector width and the cluster size.
cudaError_t launch_build_tables(const uint8_t* mask, int nb, int Hq, int Hkv, int nQblk,
                                int nKblk, int32_t* tables, int32_t* counts,
                                cudaStream_t stream) {
  // Cluster size: enough CTAs for ~CA_BUILD_CTAS_PER_SM per SM over all (mask, group) units,
  // at most 8 per cluster and at least 256 columns per CTA.
  const long long units = (long long)nb * Hkv;
  int C = (int)((CA_BUILD_CTAS_PER_SM * num_sms() + units - 1) / units);
  C = C > 8 ? 8 : C;
  const int cmax = (nKblk + 255) / 256;
  C = C > cmax ? cmax : C;
  const int cmin = (nKblk + kMaxSlab - 1) / kMaxSlab;  // slabs of at most kMaxSlab columns
  if (C < cmin) C = cmin;                              // (<= 8 for nKblk <= 65536)
  if (C < 1) C = 1;
  int slab = (nKblk + C - 1) / C;
  slab = (slab + 31) & ~31;
  if (slab > kMaxSlab) return cudaErrorInvalidValue;  // nKblk > 65536
  C = (nKblk + slab - 1) / slab;
  const uintptr_t a = reinterpret_cast<uintptr_t>(mask);
  int vec = 1;
  if (nKblk % 16 == 0 && a % 16 == 0) vec = 16;
  else if (nKblk % 4 == 0 && a % 4 == 0) vec = 4;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, Hkv, nb);
  cfg.blockDim = dim3(kBuildThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (vec == 16)
    return cudaLaunchKernelEx(&cfg, build_tables_kernel<16>, mask, Hq, Hkv, nQblk, nKblk, slab,
                              tables, counts);
  if (vec == 4)
    return cudaLaunchKernelEx(&cfg, build_tables_kernel<4>, mask, Hq, Hkv, nQblk, nKblk, slab,
                              tables, counts);
  return cudaLaunchKernelEx(&cfg, build_tables_kernel<1>, mask, Hq, Hkv, nQblk, nKblk, slab,
                            tables, counts);
}

}  // namespace ca

namespace ca {

// ---------------------------------------------------------------------------
// Bit-packed masks: bit j of 32-bit word w of a row selects KV block 32w + j.
// The union of a group is a word-wise OR over its G*nQblk rows (8x fewer bytes
// than one byte per block); one CTA per (mask, group) ORs the rows with 16-
// or 4-byte loads, then ranks the set bits with a block scan of per-thread
// popcounts and writes the ascending entries and the -1 padding.
constexpr int kBitsThreads = 256;
constexpr int kMaxBitWords = 2048;  // nKblk <= 65536

template <int VECW>  // words per load: 4 (uint4) or 1
__global__ void __launch_bounds__(kBitsThreads)
    build_tables_bits_kernel(const uint32_t* __restrict__ bits, int Hq, int Hkv, int nQblk,
                             int nKblk, int32_t* __restrict__ tables,
                             int32_t* __restrict__ counts) {
  __shared__ uint32_t uni[kMaxBitWords];
  __shared__ int warp_sum[kBitsThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x, b = blockIdx.y;
  const int G = Hq / Hkv, R = G * nQblk;
  const int W = (nKblk + 31) >> 5;
  const uint32_t* base = bits + ((size_t)b * Hq + (size_t)g * G) * (size_t)nQblk * W;
  for (int w = tid; w < W; w += kBitsThreads) uni[w] = 0u;
  __syncthreads();

  // ---- OR down the group's rows
  const int nv = W / VECW;
  int CW = 1;
  while (CW < nv && CW < kBitsThreads) CW <<= 1;
  const int RT = kBitsThreads / CW, rt = tid / CW;
  for (int v = tid % CW; v < nv; v += CW) {
    if (VECW == 4) {
      uint4 acc = make_uint4(0, 0, 0, 0);
      const uint4* p = reinterpret_cast<const uint4*>(base + (size_t)rt * W) + v;
      const size_t step = (size_t)RT * W / 4;
#pragma unroll 8
      for (int r = rt; r < R; r += RT) {
        const uint4 x = __ldcs(p);
        acc.x |= x.x; acc.y |= x.y; acc.z |= x.z; acc.w |= x.w;
        p += step;
      }
      if (acc.x) atomicOr(&uni[4 * v], acc.x);
      if (acc.y) atomicOr(&uni[4 * v + 1], acc.y);
      if (acc.z) atomicOr(&uni[4 * v + 2], acc.z);
      if (acc.w) atomicOr(&uni[4 * v + 3], acc.w);
    } else {
      uint32_t acc = 0u;
      const uint32_t* p = base + (size_t)rt * W + v;
      const size_t step = (size_t)RT * W;
#pragma unroll 8
      for (int r = rt; r < R; r += RT) {
        acc |= __ldcs(p);
        p += step;
      }
      if (acc) atomicOr(&uni[v], acc);
    }
  }
  __syncthreads();
  if (tid == 0 && (nKblk & 31)) uni[W - 1] &= (1u << (nKblk & 31)) - 1u;  // bits past nKblk
  __syncthreads();

  // ---- rank: thread t owns words [t*k, t*k + k)
  const int k = (W + kBitsThreads - 1) / kBitsThreads;
  const int w0 = min(W, tid * k), w1 = min(W, w0 + k);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(uni[w]);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kBitsThreads / 32; ++w) {
    before += (w < warp) ? warp_sum[w] : 0;
    total += warp_sum[w];
  }
  int pos = before + incl - cnt;
  int32_t* trow = tables + ((size_t)b * Hkv + g) * nKblk;
  for (int w = w0; w < w1; ++w) {
    uint32_t x = uni[w];
    while (x) {
      const int bit = __ffs(x) - 1;
      trow[pos++] = w * 32 + bit;
      x &= x - 1;
    }
  }
  for (int q = total + tid; q < nKblk; q += kBitsThreads) trow[q] = -1;
  if (tid == 0) counts[(size_t)b * Hkv + g] = total;
}

template __global__ void build_tables_bits_kernel<4>(const uint32_t*, int, int, int, int, int32_t*,
                                                     int32_t*);
template __global__ void build_tables_bits_kernel<1>(const uint32_t*, int, int, int, int, int32_t*,
                                                     int32_t*);

cudaError_t launch_build_tables_bits(const uint32_t* bits, int nb, int Hq, int Hkv, int nQblk,
                                     int nKblk, int32_t* tables, int32_t* counts,
                                     cudaStream_t stream) {
  const int W = (nKblk + 31) / 32;
  if (W > kMaxBitWords) return cudaErrorInvalidValue;
  const dim3 grid(Hkv, nb);
  if (W % 4 == 0 && (reinterpret_cast<uintptr_t>(bits) & 15u) == 0)
    build_tables_bits_kernel<4><<<grid, kBitsThreads, 0, stream>>>(bits, Hq, Hkv, nQblk, nKblk,
                                                                   tables, counts);
  else
    build_tables_bits_kernel<1><<<grid, kBitsThreads, 0, stream>>>(bits, Hq, Hkv, nQblk, nKblk,
                                                                   tables, counts);
  return cudaGetLastError();
}

}  // namespace ca
