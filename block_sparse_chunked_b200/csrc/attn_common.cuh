// attn_common.cuh — device helpers shared by the chunk-attention kernels:
// the work-unit map (sequence, KV group, 64-token query span, head slice),
// the live prefix of a unit's table, and the warp-uniform bounded wait.
#pragma once
#include <cstdint>

#include "compactattn.h"
#include "internal.h"
#include "ptx.cuh"

namespace ca {

__device__ __forceinline__ void set_flag(int32_t* err, int f) {
  if (err) atomicOr(err, f);
}

// Warp-uniform bounded wait.  Returns false (and flags / aborts) on expiry.
// A phase that has already completed is taken without reading the abort flag
// (its data is ready either way); only a wait that would block first checks
// whether another warp has given up.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const AttnParams& p,
                                          volatile int* abort_flag) {
  bool ok = mbar_try_wait(bar, parity) ||
            ((*abort_flag == 0) && mbar_wait(bar, parity, p.wait_ns));
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) {
    if ((threadIdx.x & 31) == 0 && *abort_flag == 0) {
      *abort_flag = 1;
      set_flag(p.err, CA_FLAG_TIMEOUT);
    }
  }
  return ok;
}

// Number of work units whose stage counts a persistent CTA keeps in shared memory.
constexpr int kMaxUnits = 2048;

// The sequence that owns unit u.
__device__ __forceinline__ SeqDesc seq_of(const AttnParams& p, int u) {
  if (p.seqs == nullptr) return p.seq0;
  int lo = 0, hi = p.num_seqs - 1;  // last sequence with unit_start <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seqs[mid].unit_start <= u) lo = mid;
    else hi = mid - 1;
  }
  return p.seqs[lo];
}

// Unit u -> (sequence, group, 64-token query span, head slice).  Within a
// sequence, by query span (later spans, with more causal blocks, first), or,
// with p.unit_order = 1, by group first and then by span, later spans first.
struct UnitCoord {
  SeqDesc d;
  int g, qs, hh;
};
__device__ __forceinline__ UnitCoord unit_coord(const AttnParams& p, int u) {
  UnitCoord c;
  c.d = seq_of(p, u);
  const int loc = u - c.d.unit_start;
  if (p.unit_order == 1) {
    const int per_g = c.d.nqs * p.nhalves;
    c.g = loc / per_g;
    c.qs = c.d.nqs - 1 - (loc % per_g) / p.nhalves;
    c.hh = (loc % per_g) % p.nhalves;
  } else {
    const int per_qs = p.Hkv * p.nhalves;
    c.qs = c.d.nqs - 1 - loc / per_qs;
    c.g = (loc % per_qs) / p.nhalves;
    c.hh = (loc % per_qs) % p.nhalves;
  }
  return c;
}

__device__ __forceinline__ const int32_t* table_row(const AttnParams& p, const UnitCoord& c) {
  return p.tables + (size_t)c.d.pt_off * p.Hkv + (size_t)c.g * c.d.nKblk;
}

// Live table entries of unit u: the entries whose block can hold a key visible
// to the span's last query (kb * B <= P + last token), a prefix of the
// ascending row (binary search).
__device__ __forceinline__ int unit_live(const AttnParams& p, int u) {
  const UnitCoord c = unit_coord(p, u);
  const int t_last = min(c.qs * 64 + 63, c.d.L - 1);
  const int last_kb = (c.d.P + t_last) / p.B;
  const int32_t* trow = table_row(p, c);
  int cnt = p.counts[(size_t)c.d.seq * p.Hkv + c.g];
  if (cnt < 0 || cnt > c.d.nKblk) {
    set_flag(p.err, CA_FLAG_BOUNDS);
    cnt = cnt < 0 ? 0 : c.d.nKblk;
  }
  int lo = 0, hi = cnt;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (trow[mid] <= last_kb) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// How a piece's result leaves the CTA.
enum PieceOut : int { kOutFinal = 0, kOutSplit = 1, kOutSK = 2, kOutTail = 3 };

}  // namespace ca

namespace ca {

// unit_live computed by a whole warp: a 32-way search of the ascending table
// row (each round one load per lane), about 4 rounds of dependent loads for a
// row of 65,536 entries instead of 16.  Every lane returns the count.
__device__ __forceinline__ int unit_live_warp(const AttnParams& p, const UnitCoord& c) {
  const int lane = threadIdx.x & 31;
  const int t_last = min(c.qs * 64 + 63, c.d.L - 1);
  const int last_kb = (c.d.P + t_last) / p.B;
  const int32_t* trow = table_row(p, c);
  int cnt = p.counts[(size_t)c.d.seq * p.Hkv + c.g];
  if (cnt < 0 || cnt > c.d.nKblk) {
    if (lane == 0) set_flag(p.err, CA_FLAG_BOUNDS);
    cnt = cnt < 0 ? 0 : c.d.nKblk;
  }
  // invariant: entries [0, lo) are <= last_kb, entries [hi, cnt) are greater
  int lo = 0, hi = cnt;
  while (lo < hi) {
    const int step = (hi - lo + 31) >> 5;
    const int pos = lo + lane * step;
    const bool le = pos < hi && trow[pos] <= last_kb;
    const int nle = __popc(__ballot_sync(0xffffffffu, le));  // a prefix of the probes
    if (nle == 0) {
      hi = lo;
    } else {
      const int nlo = lo + (nle - 1) * step + 1;
      hi = min(hi, lo + nle * step);
      lo = nlo;
    }
  }
  return lo;
}

}  // namespace ca

namespace ca {

// Fused mode: the unit's group table, built by the whole CTA from the
// bit-packed masks (the Q-block union and intra-group union of the abstract,
// then the compaction) into shared memory: fent[0 .. count) ascending,
// followed (at fent + 2048) by the group's union bit set (mask_words words)
// and the count.  Returns the count.
constexpr int kMaxFusedWords = 64;  // nKblk <= 2048
static __device__ int fused_group_table(const AttnParams& p, const UnitCoord& uc, int32_t* fent,
                                 int nthreads) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = p.mask_words;
  uint32_t* uni = reinterpret_cast<uint32_t*>(fent + kMaxFusedWords * 32);
  for (int w = tid; w < W; w += nthreads) uni[w] = 0u;
  __syncthreads();
  // OR down the group's G * nQblk rows: thread -> (vector v of a row, rows r,
  // r + RT, ...), 16-byte loads when the rows allow, several loads in flight
  const int R = p.G * p.nQblk_mask;
  const uint32_t* base = p.mask_bits + (size_t)uc.g * R * W;
  const bool vec4 = (W % 4) == 0 && (reinterpret_cast<uintptr_t>(p.mask_bits) & 15u) == 0;
  const int NV = vec4 ? W / 4 : W;
  const int RT = nthreads / NV;
  if (tid < RT * NV) {
    const int v = tid % NV;
    if (vec4) {
      uint4 acc = make_uint4(0u, 0u, 0u, 0u);
      const uint4* rowp = reinterpret_cast<const uint4*>(base) + v;
#pragma unroll 8
      for (int r = tid / NV; r < R; r += RT) {
        const uint4 x = __ldg(rowp + (size_t)r * NV);
        acc.x |= x.x;
        acc.y |= x.y;
        acc.z |= x.z;
        acc.w |= x.w;
      }
      if (acc.x) atomicOr(&uni[4 * v], acc.x);
      if (acc.y) atomicOr(&uni[4 * v + 1], acc.y);
      if (acc.z) atomicOr(&uni[4 * v + 2], acc.z);
      if (acc.w) atomicOr(&uni[4 * v + 3], acc.w);
    } else {
      uint32_t acc = 0u;
#pragma unroll 8
      for (int r = tid / NV; r < R; r += RT) acc |= __ldg(base + (size_t)r * W + v);
      if (acc) atomicOr(&uni[v], acc);
    }
  }
  __syncthreads();
  if (tid == 0 && (uc.d.nKblk & 31)) uni[W - 1] &= (1u << (uc.d.nKblk & 31)) - 1u;
  __syncthreads();
  // compaction by warp 0: lane l ranks words 2l and 2l + 1
  int* total = reinterpret_cast<int*>(uni + kMaxFusedWords);
  if (warp == 0) {
    const int w0 = 2 * lane;
    const uint32_t x0 = w0 < W ? uni[w0] : 0u, x1 = w0 + 1 < W ? uni[w0 + 1] : 0u;
    const int cnt = __popc(x0) + __popc(x1);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - cnt;
    for (uint32_t x = x0; x; x &= x - 1) fent[pos++] = w0 * 32 + __ffs(x) - 1;
    for (uint32_t x = x1; x; x &= x - 1) fent[pos++] = (w0 + 1) * 32 + __ffs(x) - 1;
    if (lane == 31) *total = incl;
  }
  __syncthreads();
  return *total;
}

}  // namespace ca
