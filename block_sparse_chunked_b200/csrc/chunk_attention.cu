// chunk_attention.cu — chunked-prefill attention over the selected KV blocks
// of a paged cache, for sm_100a (tcgen05 tensor cores, TMEM, TMA).
//
// "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection", Abstract: every query of a GQA group reads exactly the KV
// blocks of its group's table, in place in the paged cache, with no KV
// compaction.
//
// Work unit = (KV group g, 64-token query span qs, head slice hh, KV split).
// The unit's rows are the span's 64 tokens for up to four query heads of the
// group, stacked into NT = 1 or 2 tensor-core tiles of 128 rows (two heads per
// tile).  All rows of a unit share the group's table, so every KV block
// fetched from HBM/L2 feeds 2*NT MMAs.  The blocks a span may see are a prefix
// of the sorted table (entries whose block holds a position <= the span's last
// query), and only the last one or two of them (those past the span's first
// query position: for a block-aligned chunk, the diagonal block) need a
// token-level causal mask.
//
// One CTA per unit (1 CTA / SM: it holds all 512 TMEM columns):
//   warp 0      TMA producer: Q tiles once, then per stage the K and V pages
//               of up to 128 keys (one or two table entries), looked up
//               through tables -> page_table -> physical page (in place);
//   warp 1      TMEM allocator and tcgen05.mma issuer (one thread):
//               S_t = Q_t K^T (SS) and O_t += P_t V (TS: P read from TMEM);
//   warps 4..   one softmax warpgroup per tile: each thread owns one row,
//               loads its S row from TMEM, applies scale and the diagonal
//               causal mask, keeps the running max / sum (the max is only
//               moved when it grows by more than 2^8, which keeps the result
//               exact and skips most O rescales), writes P as bf16 back over
//               S in TMEM, and finally normalises O and writes O / LSE (or
//               the fp32 partials of a KV split).
// TMEM columns: O_0 [0,128) O_1 [128,256) S_0 [256,384) S_1 [384,512).
// Every pipeline wait is bounded; on expiry the CTA records CA_FLAG_TIMEOUT
// and unwinds instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "compactattn.h"
#include "attn_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace ca {

constexpr int kStageKeys = 128;



// QSPLIT: Q is given as two bf16 terms (hi + lo) of an fp32 input and
// S = Q_hi K^T + Q_lo K^T, which removes the rounding error of Q (the error
// term shared by all keys of a row); used for fp32 inputs.
//
// KV8: K/V pages hold E4M3 bytes; TMA brings a stage's K and V bytes into two
// staging halves, warps 2-3 widen them to f16 into the swizzled operand ring, and
// the MMAs run kind::f16 with f16 operands (Q converted to f16, P written as
// f16).  The per-page scales are applied in the softmax.
template <int D, int NT, bool QSPLIT, bool KV8 = false>
struct Smem {
  static constexpr int kQTerms = QSPLIT ? 2 : 1;
  static constexpr int kChunkBytes = 128 * 128;         // 128 rows x 128 B (64 16-bit)
  static constexpr int kQTile = 128 * D * 2;            // one 128-row Q tile
  static constexpr int kKV = kStageKeys * D * 2;        // one stage of K (or V)
  static constexpr int kStg = KV8 ? 2 * kStageKeys * D : 0;  // E4M3 K + V of one stage
  // K/V ring depth: two stages unless the split Q tiles leave room for one only
  static constexpr int kNS =
      KV8 ? 2 : ((kQTerms * NT * kQTile + 4 * kKV <= 200 * 1024) ? 2 : 1);
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQTerms * NT * kQTile;
  static constexpr int kVOff = kKOff + kNS * kKV;
  static constexpr int kStgOff = kVOff + kNS * kKV;
  static constexpr int kBarOff = kStgOff + kStg;
  // barriers: q_full, full_k[NS], full_v[NS], empty_k[NS], empty_v[NS],
  //           s_full[2], p_full[2], o_done, drain, q_free
  //           (+ KV8: stg_full[2], stg_empty[2] for the K and V staging halves)
  static constexpr int kNumBars = 1 + 4 * kNS + 2 + 2 + 3 + (KV8 ? 4 : 0);
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // persistent schedule: per-unit live entries, prefix of stage counts, warp sums
  // (not used with E4M3 pages, which run one CTA per unit or KV splits)
  static constexpr int kSchedOff = kMiscOff + 64;
  static constexpr int kBytes = kSchedOff + (KV8 ? 0 : (2 * 2048 + 1 + 32) * 4);
  static constexpr int kAlloc = kBytes + 1024;          // slack for 1024-B alignment
};

template <int D, int NT, bool QSPLIT, bool KV8>
__global__ void __launch_bounds__(128 + NT * 128, 1)
    chunk_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmQlo,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using S = Smem<D, NT, QSPLIT, KV8>;
  constexpr int kNS = S::kNS;
  constexpr int KCH = D / 64;  // 64-element (128-byte) chunks along head_dim
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bars = sbase + S::kBarOff;
  const uint32_t q_full = bars;
  auto full_k = [&](int s) { return bars + 8u * (1 + s); };
  auto full_v = [&](int s) { return bars + 8u * (1 + kNS + s); };
  auto empty_k = [&](int s) { return bars + 8u * (1 + 2 * kNS + s); };
  auto empty_v = [&](int s) { return bars + 8u * (1 + 3 * kNS + s); };
  auto s_full = [&](int t) { return bars + 8u * (1 + 4 * kNS + t); };
  auto p_full = [&](int t) { return bars + 8u * (3 + 4 * kNS + t); };
  const uint32_t o_done = bars + 8u * (5 + 4 * kNS);
  const uint32_t drain = bars + 8u * (6 + 4 * kNS);
  const uint32_t q_free = bars + 8u * (7 + 4 * kNS);
  // KV8 only: staging half h (0 = K, 1 = V) loaded / widened
  auto stg_full = [&](int h) { return bars + 8u * (8 + 4 * kNS + h); };
  auto stg_empty = [&](int h) { return bars + 8u * (10 + 4 * kNS + h); };
  int* misc = reinterpret_cast<int*>(sm + S::kMiscOff);
  // misc[0] tmem base, [1] live entries (one-piece mode), [2] first stage,
  // [3] last stage (exclusive), [4] live entries of the fused table (thread 0
  // only), [5] abort
  volatile int* abort_flag = misc + 5;
  int* sk_live = reinterpret_cast<int*>(sm + S::kSchedOff);  // [kMaxUnits] (persistent)
  int* sk_pref = sk_live + kMaxUnits;                         // [kMaxUnits + 1]

  // A batched call's grid is an upper bound on its units: surplus CTAs leave
  // before touching shared memory, barriers or TMEM.
  if (p.n_units_dev && !p.persistent && (int)(blockIdx.x / p.n_splits) >= *p.n_units_dev) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int spb = kStageKeys / p.B;  // pages per stage
  const int nthreads = 128 + NT * 128;

  // ---- work: one piece (one-piece mode) or a contiguous range of all
  // units' stages (persistent mode)
  if (threadIdx.x == 0) misc[5] = 0;
  // fused mode keeps the group table here (the persistent schedule is not used then)
  int32_t* fent = sk_live;
  if (!p.persistent) {
    if (p.mask_bits) {
      const int u = blockIdx.x / p.n_splits;
      const UnitCoord uc = unit_coord(p, u);
      const int cnt = fused_group_table(p, uc, fent, nthreads);
      if (uc.qs == 0 && uc.hh == 0 && blockIdx.x % p.n_splits == 0) {  // one CTA per group
        if (p.tables_out) {
          int32_t* trow_out = p.tables_out + (size_t)uc.g * uc.d.nKblk;
          for (int e = threadIdx.x; e < uc.d.nKblk; e += nthreads)
            trow_out[e] = e < cnt ? fent[e] : -1;
        }
        if (threadIdx.x == 0 && p.counts_out) p.counts_out[uc.g] = cnt;
      }
      if (threadIdx.x == 0) {
        const int t_last = min(uc.qs * 64 + 63, uc.d.L - 1);
        const int last_kb = (uc.d.P + t_last) / p.B;
        int lo = 0, hi = cnt;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (fent[mid] <= last_kb) lo = mid + 1;
          else hi = mid;
        }
        misc[4] = lo;
      }
    }
    if (threadIdx.x == 0) {
      const int u = blockIdx.x / p.n_splits, split = blockIdx.x % p.n_splits;
      const int live = p.mask_bits ? misc[4] : unit_live(p, u);
      const int nst = (live + spb - 1) / spb;
      misc[1] = live;
      misc[2] = (int)((long long)split * nst / p.n_splits);
      misc[3] = (int)((long long)(split + 1) * nst / p.n_splits);
    }
  } else {
    // every CTA derives the same schedule: stage counts of all units, prefix sums
    for (int u = threadIdx.x; u < p.n_units; u += nthreads) sk_live[u] = unit_live(p, u);
    __syncthreads();
    // block-wide exclusive scan of the stage counts: each thread a run of units
    const int per = (p.n_units + nthreads - 1) / nthreads;
    const int u0 = min(p.n_units, threadIdx.x * per), u1 = min(p.n_units, u0 + per);
    int run = 0;
    for (int u = u0; u < u1; ++u) run += (sk_live[u] + spb - 1) / spb;
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int* wsum = sk_pref + kMaxUnits + 1;  // scratch after the prefix array: [warps]
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wsum[w];
    int acc = base + incl - run;
    for (int u = u0; u < u1; ++u) {
      sk_pref[u] = acc;
      acc += (sk_live[u] + spb - 1) / spb;
    }
    if (threadIdx.x == nthreads - 1) sk_pref[p.n_units] = base + incl;
    __syncthreads();
    if (blockIdx.x == 0)
      for (int u = threadIdx.x; u <= p.n_units; u += nthreads) p.sk_sched[u] = sk_pref[u];
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(full_k(s), KV8 ? 2 : 1);  // KV8: the two widening warps arrive
      mbar_init(full_v(s), KV8 ? 2 : 1);
      mbar_init(empty_k(s), 1);
      mbar_init(empty_v(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 4);  // one arrival per softmax warp
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    if (KV8) {
      for (int h = 0; h < 2; ++h) {
        mbar_init(stg_full(h), 1);
        mbar_init(stg_empty(h), 2);
      }
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + S::kMiscOff, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)misc[0];

  // Visit this CTA's pieces in order: fn(unit, live entries, first stage,
  // end stage, output kind, partial slot).  Every role walks the same list.
  auto for_each_piece = [&](auto&& fn) {
    if (!p.persistent) {
      const int split = blockIdx.x % p.n_splits;
      fn(blockIdx.x / p.n_splits, misc[1], misc[2], misc[3],
         p.n_splits > 1 ? kOutSplit : kOutFinal, split);
      return;
    }
    const long long T = sk_pref[p.n_units];
    const int P = p.sk_ctas, c = blockIdx.x;
    // units without any stage: their rows are written by CTA (u mod P)
    for (int u = c; u < p.n_units; u += P)
      if (sk_pref[u + 1] == sk_pref[u]) fn(u, sk_live[u], 0, 0, kOutFinal, 0);
    const int r0 = (int)(T * c / P), r1 = (int)(T * (c + 1) / P);
    if (r1 <= r0) return;
    int lo = 0, hi = p.n_units;  // first unit with pref[u + 1] > r0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sk_pref[mid + 1] > r0) hi = mid;
      else lo = mid + 1;
    }
    bool first = true;
    for (int u = lo; u < p.n_units && sk_pref[u] < r1; ++u) {
      const int a = max(r0, sk_pref[u]) - sk_pref[u];
      const int b = min(r1, sk_pref[u + 1]) - sk_pref[u];
      if (b <= a) continue;
      const bool whole = a == 0 && b == sk_pref[u + 1] - sk_pref[u];
      fn(u, sk_live[u], a, b, whole ? kOutFinal : kOutSK, first ? 2 * c : 2 * c + 1);
      first = false;
    }
  };

  if (warp == 0) {
    // ================================================================ producer
    // The whole warp runs the loop: lane i prefetches table entry i of the next
    // group of 32 and its page id, so the dependent lookups tables ->
    // page_table are off the per-stage path; one elected lane issues copies.
    const uint64_t pol = policy_evict_last();
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      if (QSPLIT) prefetch_tmap(&tmQlo);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    int gj = 0, pn = 0;  // global stage counter, non-empty piece counter
    bool ok = true;
    for_each_piece([&](int u, int live, int s0, int s1, int, int) {
      if (s1 <= s0 || !ok) return;
      const UnitCoord uc = unit_coord(p, u);
      const int32_t* trow = p.mask_bits ? fent : table_row(p, uc);
      if (pn > 0) ok = wait_warp(q_free, (pn - 1) & 1, p, abort_flag);
      if (ok && lane == 0) {
        mbar_expect_tx(q_full, S::kQTerms * NT * 128 * D * 2);
        for (int q = 0; q < S::kQTerms; ++q)
          for (int t = 0; t < NT; ++t)
            for (int s = 0; s < 2; ++s) {
              int hl = uc.hh * p.HPU + 2 * t + s;  // head within the group
              const int hcap = min(p.G - 1, uc.hh * p.HPU + p.HPU - 1);
              hl = min(hl, hcap);
              const int head = uc.g * p.G + hl;
              for (int c = 0; c < KCH; ++c)
                tma_load_3d(sbase + S::kQOff + (q * NT + t) * S::kQTile + c * S::kChunkBytes +
                                s * 64 * 128,
                            q ? &tmQlo : &tmQ, q_full, c * 64, head, uc.d.q_start + uc.qs * 64);
            }
      }
      const int e_begin = s0 * spb, e_end = min(live, s1 * spb);
      int pg_cache = 0, cache_base = -32;
      for (int stage = s0; stage < s1 && ok; ++stage, ++gj) {
        const int slot = gj % kNS, round = gj / kNS;
        const int npg = min(spb, live - stage * spb);
        const uint32_t bytes = (uint32_t)npg * p.B * D * 2;
        int page[2] = {0, 0};
        for (int pi = 0; pi < npg; ++pi) {
          const int e = stage * spb + pi;
          if (e >= cache_base + 32) {  // refill: 32 entries, one per lane
            cache_base = e;
            const int my = e + lane;
            int pg = 0;
            if (my < e_end && my >= e_begin) {
              int kb = trow[my];
              if (kb < 0 || kb >= uc.d.nKblk) {
                set_flag(p.err, CA_FLAG_BOUNDS);
                kb = 0;
              }
              pg = p.page_table[uc.d.pt_off + kb];
              if (pg < 0 || pg >= p.num_pages) {
                set_flag(p.err, CA_FLAG_BOUNDS);
                pg = 0;
              }
            }
            pg_cache = pg;
          }
          page[pi] = __shfl_sync(0xffffffffu, pg_cache, e - cache_base);
        }
        if (KV8) {
          // E4M3 bytes of the stage's pages into the staging halves (K, then
          // V), each as soon as the widening warps are done with its previous
          // contents, so one half loads while the other is widened
          const uint32_t b8 = (uint32_t)npg * p.B * D;
          for (int h = 0; h < 2 && ok; ++h) {
            if (gj > 0) ok = wait_warp(stg_empty(h), (gj - 1) & 1, p, abort_flag);
            if (!ok) break;
            mbar_expect_tx_w(stg_full(h), b8);
            for (int pi = 0; pi < npg; ++pi)
              tma_load_4d_w(sbase + S::kStgOff + h * kStageKeys * D + pi * p.B * D,
                            h ? &tmV : &tmK, stg_full(h), 0, 0, uc.g, page[pi], pol);
          }
          continue;
        }
        if (round > 0) ok = wait_warp(empty_k(slot), (round - 1) & 1, p, abort_flag);
        if (ok) {
          mbar_expect_tx_w(full_k(slot), bytes);
          for (int pi = 0; pi < npg; ++pi)
            for (int c = 0; c < KCH; ++c)
              tma_load_4d_w(sbase + S::kKOff + slot * S::kKV + c * S::kChunkBytes + pi * p.B * 128,
                            &tmK, full_k(slot), c * 64, 0, uc.g, page[pi], pol);
        }
        if (ok && round > 0) ok = wait_warp(empty_v(slot), (round - 1) & 1, p, abort_flag);
        if (ok) {
          mbar_expect_tx_w(full_v(slot), bytes);
          for (int pi = 0; pi < npg; ++pi)
            for (int c = 0; c < KCH; ++c)
              tma_load_4d_w(sbase + S::kVOff + slot * S::kKV + c * S::kChunkBytes + pi * p.B * 128,
                            &tmV, full_v(slot), c * 64, 0, uc.g, page[pi], pol);
        }
      }
      ++pn;
    });
    if (lane == 0) {
      // Do not leave with copies in flight: the last stages' loads must land.
      if (KV8) {
        if (gj > 0) {
          mbar_wait(stg_full(0), (gj - 1) & 1, p.wait_ns);
          mbar_wait(stg_full(1), (gj - 1) & 1, p.wait_ns);
        }
      } else {
        for (int G = max(0, gj - kNS); G < gj; ++G) {
          mbar_wait(full_k(G % kNS), (G / kNS) & 1, p.wait_ns);
          mbar_wait(full_v(G % kNS), (G / kNS) & 1, p.wait_ns);
        }
      }
      if (pn > 0) mbar_wait(q_full, (pn - 1) & 1, p.wait_ns);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // The whole warp runs this loop (addresses stay warp-uniform); one elected
    // lane issues each tcgen05.mma / commit.
    // Descriptors differ per MMA only in the start-address field (address >> 4
    // in bits 0-13): build each operand's descriptor once and add the
    // compile-time byte offset >> 4 per K-step.
    constexpr uint32_t kIdescPV = KV8 ? idesc_f16(128, D, 1) : idesc_bf16(128, D, 1);
    constexpr uint32_t kIdescS128 = KV8 ? idesc_f16(128, 128, 0) : idesc_bf16(128, 128, 0);
    constexpr uint32_t kIdescS64 = KV8 ? idesc_f16(128, 64, 0) : idesc_bf16(128, 64, 0);
    uint64_t qdesc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) qdesc[t] = smem_desc_sw128(sbase + S::kQOff + t * S::kQTile, 16, 1024);
    const uint64_t kdesc0 = smem_desc_sw128(sbase + S::kKOff, 16, 1024);
    const uint64_t vdesc0 = smem_desc_sw128(sbase + S::kVOff, S::kChunkBytes, 1024);
    int gj = 0, pn = 0;
    bool ok = true;
    for_each_piece([&](int, int live, int s0, int s1, int, int) {
      if (s1 <= s0 || !ok) return;
      const int n = s1 - s0;
      auto keys_of = [&](int j) { return min(spb, live - (s0 + j) * spb) * p.B; };
      auto issue_s = [&](int t, int j) {
        const uint64_t kd = kdesc0 + (uint64_t)((((gj + j) % kNS) * S::kKV) >> 4);
        const uint32_t idesc = keys_of(j) == 128 ? kIdescS128 : kIdescS64;
        const uint32_t dt = tmem + 256 + t * 128;
#pragma unroll
        for (int q = 0; q < S::kQTerms; ++q)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * S::kChunkBytes + (kk & 3) * 32) >> 4;
            mma_ss_w(dt, qdesc[t] + (uint64_t)(((q * NT * S::kQTile) >> 4) + off), kd + off, idesc,
                     (q > 0 || kk > 0) ? 1u : 0u);
          }
      };
      auto issue_pv = [&](int t, int j) {
        const uint64_t vd = vdesc0 + (uint64_t)((((gj + j) % kNS) * S::kKV) >> 4);
        const uint32_t dt = tmem + t * 128;
        const uint32_t at = tmem + 256 + t * 128;
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        if (keys_of(j) == 128) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(dt, at + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV, kk > 0 ? 1u : acc0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts_w(dt, at + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV, kk > 0 ? 1u : acc0);
        }
      };
      ok = wait_warp(q_full, pn & 1, p, abort_flag) &&
           wait_warp(full_k(gj % kNS), (gj / kNS) & 1, p, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit_w(s_full(0));
        if (NT == 2) {
          issue_s(1, 0);
          mma_commit_w(s_full(1));
        }
        mma_commit_w(empty_k(gj % kNS));
      }
      for (int j = 0; j < n && ok; ++j) {
        const int G = gj + j, slot = G % kNS;
        ok = wait_warp(p_full(0), G & 1, p, abort_flag) &&
             wait_warp(full_v(slot), (G / kNS) & 1, p, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, j);
        const bool more = j + 1 < n;
        if (more) {
          ok = wait_warp(full_k((G + 1) % kNS), ((G + 1) / kNS) & 1, p, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, j + 1);
          mma_commit_w(s_full(0));
        }
        if (NT == 2) {
          ok = wait_warp(p_full(1), G & 1, p, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, j);
        }
        mma_commit_w(empty_v(slot));
        if (more) {
          if (NT == 2) {
            issue_s(1, j + 1);
            mma_commit_w(s_full(1));
          }
          mma_commit_w(empty_k((G + 1) % kNS));
        }
      }
      if (ok) {
        mma_commit_w(o_done);  // this piece's O is complete
        mma_commit_w(q_free);  // and no MMA reads its Q any more
      }
      gj += n;
      ++pn;
    });
    // every MMA issued by this warp has finished before TMEM is released
    mma_commit_w(drain);
    mbar_wait(drain, 0, p.wait_ns);
  } else if (KV8 && (warp == 2 || warp == 3)) {
    // ================================================================ E4M3 -> f16
    // Widen the staged bytes of each stage into the swizzled f16 operand ring
    // (same layout the TMA gives bf16 pages: 64-element chunks of 128 rows x
    // 128 B, 16-byte units XOR-swizzled by row), K then V.
    const int ct = threadIdx.x - 64;  // 0 .. 63
    int gj = 0;
    bool ok = true;
    // Thread ct always handles the same 16-byte column chunk q of rows r0,
    // r0 + RS, ...; RS is a multiple of 8, so the row's swizzle phase (r & 7)
    // and hence both 16-byte destination units are fixed per thread.
    constexpr int CPR = D / 16;   // 16-byte chunks per E4M3 row
    constexpr int RS = 64 / CPR;  // rows between a thread's chunks (8 or 16)
    static_assert(RS % 8 == 0, "swizzle phase must repeat");
    const int q = ct % CPR, r0 = ct / CPR;
    const int u = (q & 3) * 2;  // first 16-byte unit of these 16 elements in a row
    const uint32_t dst_lo = (q >> 2) * S::kChunkBytes + ((u ^ (r0 & 7)) << 4);
    const uint32_t dst_hi = (q >> 2) * S::kChunkBytes + (((u + 1) ^ (r0 & 7)) << 4);
    // E4M3 byte b -> f16 bits (sign << 15) | ((b & 0x7F) << 7): that f16 is
    // decode(b) / 256 for every non-NaN code, subnormals included (the f16
    // exponent bias is 8 above E4M3's and E4M3 subnormals land on f16
    // subnormals); the 256 is folded into the page scales.  With a pair of bytes
    // placed in the high byte of each 16-bit half (t), y = t >> 1 puts the
    // magnitude at bits 7..13 and the sign at bit 14, and y + (y & 0x4000)
    // moves the sign to bit 15.  Integer ops only, leaving the SFU to the
    // exponentials.
    auto pair = [](uint32_t w, uint32_t sel) {
      const uint32_t y = __byte_perm(w, 0u, sel) >> 1;
      return y + (y & 0x40004000u);
    };
    auto widen = [&](uint32_t src_off, uint32_t dst_off, int rows) {
      const uint8_t* src = sm + src_off + q * 16;
      uint8_t* dst = sm + dst_off;
      for (int r = r0; r < rows; r += RS) {
        const uint4 x = *reinterpret_cast<const uint4*>(src + r * D);
        uint8_t* rowp = dst + r * 128;
        *reinterpret_cast<uint4*>(rowp + dst_lo) =
            make_uint4(pair(x.x, 0x1404), pair(x.x, 0x3424), pair(x.y, 0x1404), pair(x.y, 0x3424));
        *reinterpret_cast<uint4*>(rowp + dst_hi) =
            make_uint4(pair(x.z, 0x1404), pair(x.z, 0x3424), pair(x.w, 0x1404), pair(x.w, 0x3424));
      }
      fence_proxy_async_smem();  // the tensor cores read these bytes next
      __syncwarp();
    };
    for_each_piece([&](int, int live, int s0, int s1, int, int) {
      for (int stage = s0; stage < s1 && ok; ++stage, ++gj) {
        const int slot = gj % kNS, round = gj / kNS;
        const int rows = min(spb, live - stage * spb) * p.B;
        ok = wait_warp(stg_full(0), gj & 1, p, abort_flag);
        if (ok && round > 0) ok = wait_warp(empty_k(slot), (round - 1) & 1, p, abort_flag);
        if (!ok) break;
        widen(S::kStgOff, S::kKOff + slot * S::kKV, rows);
        if (lane == 0) {
          mbar_arrive(full_k(slot));
          mbar_arrive(stg_empty(0));
        }
        ok = wait_warp(stg_full(1), gj & 1, p, abort_flag);
        if (ok && round > 0) ok = wait_warp(empty_v(slot), (round - 1) & 1, p, abort_flag);
        if (!ok) break;
        widen(S::kStgOff + kStageKeys * D, S::kVOff + slot * S::kKV, rows);
        if (lane == 0) {
          mbar_arrive(full_v(slot));
          mbar_arrive(stg_empty(1));
        }
      }
    });
  } else if (warp >= 4) {
    // ================================================================ softmax / epilogue
    const int t = (warp - 4) >> 2;
    const int row = threadIdx.x & 127;
    const int sub = row >> 6;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + 256 + t * 128;
    const uint32_t tO = tmem + lane_off + t * 128;
    int gj = 0, pn = 0;
    bool ok = true;
    for_each_piece([&](int u, int live, int s0, int s1, int out, int slot) {
      const UnitCoord uc = unit_coord(p, u);
      const int t0 = uc.qs * 64;
      const int tl = t0 + (row & 63);     // token within the chunk
      const int tok = uc.d.q_start + tl;  // row of Q / O
      const int hl_raw = uc.hh * p.HPU + 2 * t + sub;
      const bool valid_row = (2 * t + sub) < p.HPU && hl_raw < p.G && tl < uc.d.L;
      const int head = uc.g * p.G + min(hl_raw, p.G - 1);
      const int32_t* trow = p.mask_bits ? fent : table_row(p, uc);
      // Token-level causal mask: only blocks that hold a key later than the
      // span's first query (kb >= (P + t0) / B) need it; in the ascending
      // table they are the last live entries, from mask_e on.
      const int kb_m0 = (uc.d.P + t0) / p.B;
      int mask_e = live;
      while (mask_e > 0 && trow[mask_e - 1] >= kb_m0) --mask_e;
      // those are consecutive blocks (at most the two the span's positions fall
      // in): their first key positions
      const int kposA = mask_e < live ? trow[mask_e] * p.B : 0;
      const int kposB = kposA + p.B;
      const int qpos = uc.d.P + tl;  // this row's position: keys j <= qpos are visible
      const int n = s1 - s0;
      float m_used = -INFINITY, l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
      for (int j = 0; j < n && ok; ++j) {
        const int stage = s0 + j, G = gj + j;
        const int npg = min(spb, live - stage * spb);
        const int nvalid = npg * p.B;
        const bool mask_stage = stage * spb + npg > mask_e;
        float2 scl_a = make_float2(1.f, 1.f), scl_b = scl_a;  // KV8: (K, V) scales per half
        if (KV8) {
          const float2* es = p.escale + (size_t)uc.g * uc.d.nKblk + stage * spb;
          scl_a = es[0];
          scl_b = npg > 1 ? es[1] : scl_a;
        }
        ok = wait_warp(s_full(t), G & 1, p, abort_flag);
        if (!ok) break;
        tc_fence_after();
        // One TMEM pass: the row's scores (raw Q.K) into registers.
        float sr[kStageKeys];
        tmem_ld64f(tS, sr);
        if (nvalid > 64) tmem_ld64f(tS + 64, sr + 64);
        tmem_wait_ld();
        if (nvalid <= 64) {
#pragma unroll
          for (int c = 64; c < kStageKeys; ++c) sr[c] = -INFINITY;
        }
        if (mask_stage) {  // keys after this row's position -> -inf
          // From the stage's first page that needs the mask, page pm, the key of
          // column c >= pm * B is (its block) * B + (c - pm * B).
          const int e0 = stage * spb;
          const int pm = max(0, mask_e - e0);
          const int cm0 = pm * p.B;
          const int lim = qpos - (e0 + pm > mask_e ? kposB : kposA);  // visible while c - cm0 <= lim
#pragma unroll
          for (int c = 0; c < kStageKeys; ++c)
            if (c >= cm0 && (c - cm0) > lim) sr[c] = -INFINITY;
        }
        // row max of the raw scores (scale > 0 commutes with max)
        float mx;
        float scA = p.scale_log2, scB = p.scale_log2, lbA = 0.f, lbB = 0.f;
        if (KV8) {
          // E4M3 pages: the log2-domain score of a key of page P is
          // s * scale * sK_P, and its weight enters PV multiplied by sV_P, so the
          // exponent carries + log2(sV_P) (the row sum divides it out again)
          scA *= scl_a.x;
          scB *= scl_b.x;
          lbA = __log2f(scl_a.y);
          lbB = __log2f(scl_b.y);
          float ha = max3(sr[0], sr[1], sr[2]), hb = max3(sr[64], sr[65], sr[66]);
#pragma unroll
          for (int c = 3; c < 63; c += 2) {
            ha = max3(ha, sr[c], sr[c + 1]);
            hb = max3(hb, sr[64 + c], sr[64 + c + 1]);
          }
          ha = fmaxf(ha, sr[63]);
          hb = fmaxf(hb, sr[127]);
          mx = fmaxf(ha * scA + lbA, hb * scB + lbB);
        } else {
          float mx0 = max3(sr[0], sr[1], sr[2]);
          float mx1 = max3(sr[3], sr[4], sr[5]);
#pragma unroll
          for (int c = 6; c < kStageKeys - 2; c += 4) {
            mx0 = max3(mx0, sr[c], sr[c + 1]);
            mx1 = max3(mx1, sr[c + 2], sr[c + 3]);
          }
          mx = max3(mx0, mx1, fmaxf(sr[kStageKeys - 2], sr[kStageKeys - 1])) * p.scale_log2;
        }
        const float m_new = fmaxf(m_used, mx);
        const bool need = (m_new != -INFINITY) && (m_new > m_used + 8.0f);
        float alpha = 1.f;
        if (need) {
          alpha = ex2(m_used - m_new);  // 0 when m_used == -inf
          l0 *= alpha;
          l1 *= alpha;
          l2 *= alpha;
          l3 *= alpha;
          m_used = m_new;
        }
        const float nm = (m_used == -INFINITY) ? 0.f : -m_used;
        if (KV8) {
          // per half: p' = 2^(s * scale * sK - m + log2 sV) = sV * p, packed as f16
          // for the f16 PV; the row sum takes sum(p') / sV = sum(p)
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int c = 0; c < kStageKeys / 32; ++c) {
            if (c * 32 < nvalid) {
              const float sc = c < 2 ? scA : scB;
              const float bias = (c < 2 ? lbA : lbB) + nm;
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float x0, x1;
                ffma2(x0, x1, sr[c * 32 + 2 * i], sr[c * 32 + 2 * i + 1], sc, sc, bias, bias);
                const float e0 = ex2(x0), e1 = ex2(x1);
                if (c < 2) fadd2(a0, a1, e0, e1);
                else fadd2(a2, a3, e0, e1);
                pk[i] = pack_f16x2(e0, e1);
              }
              tmem_st16(tS + c * 16, pk);
            }
          }
          l0 += (a0 + a1) * __frcp_rn(scl_a.y);
          l2 += (a2 + a3) * __frcp_rn(scl_b.y);
        } else {
          const float sc = p.scale_log2;
          // p = 2^(s*scale - m): packed FMA, then ex2; fp32 row sum before the bf16 rounding
#pragma unroll
          for (int c = 0; c < kStageKeys / 32; ++c) {
            if (c * 32 < nvalid) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float x0, x1;
                ffma2(x0, x1, sr[c * 32 + 2 * i], sr[c * 32 + 2 * i + 1], sc, sc, nm, nm);
                const float e0 = ex2(x0), e1 = ex2(x1);
                if (i & 1) fadd2(l2, l3, e0, e1);  // two independent sum chains
                else fadd2(l0, l1, e0, e1);
                pk[i] = pack_bf16x2(e0, e1);
              }
              tmem_st16(tS + c * 16, pk);
            }
          }
        }
        // O still holds the sum over earlier stages at the old max: bring it to the new one
        if (__any_sync(0xffffffffu, need) && j > 0) {
          uint32_t r[32];
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(t));
      }
      // ---- epilogue of the piece
      const bool ran = ok && n > 0;
      bool have_o = false;
      if (ran) {
        have_o = wait_warp(o_done, pn & 1, p, abort_flag);
        ok = have_o;
        if (have_o) tc_fence_after();
      }
      const float l = (l0 + l1) + (l2 + l3);
      const bool have = have_o && l > 0.f;
      const float inv = have ? 1.f / l : 0.f;
      const float lse = have ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      uint32_t r[32];
      for (int c = 0; c < D / 32; ++c) {
        if (have_o) {
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        if (!valid_row) continue;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = have ? __uint_as_float(r[i]) * inv : 0.f;
        float* fdst = nullptr;
        if (out == kOutSplit)
          fdst = p.Opart + (((size_t)slot * p.L + tok) * p.Hq + head) * D + c * 32;
        else if (out == kOutSK)
          fdst = p.Osk + ((size_t)slot * (NT * 128) + t * 128 + row) * D + c * 32;
        else if (p.out_f32)
          fdst = reinterpret_cast<float*>(p.O) + ((size_t)tok * p.Hq + head) * D + c * 32;
        if (fdst) {
          float4* dst = reinterpret_cast<float4*>(fdst);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.O) +
                                                ((size_t)tok * p.Hq + head) * D + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
        }
      }
      if (valid_row) {
        if (out == kOutSplit) p.LSEpart[((size_t)slot * p.Hq + head) * p.L + tok] = lse;
        else if (out == kOutSK) p.LSEsk[(size_t)slot * (NT * 128) + t * 128 + row] = lse;
        else p.LSE[(size_t)head * p.L + tok] = lse;
      }
      if (n > 0) {
        gj += n;
        ++pn;
      }
    });
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Persistent mode: merge the pieces of every unit that more than one CTA
// worked on.  Block (u, r8) handles rows [8*r8, 8*r8 + 8) of unit u, one warp
// per row (lane = D/32 consecutive columns, coalesced).  The pieces sit in
// consecutive CTAs of the stage ranges, and their partial slots follow from
// the same schedule the attention kernel used.
template <int D, int NT>
__global__ void __launch_bounds__(256)
    sk_combine_kernel(const AttnParams p) {
  const int u = blockIdx.x;
  const int32_t* pref = p.sk_sched;
  const long long T = pref[p.n_units];
  const int P = p.sk_ctas;
  const long long a = pref[u], b = pref[u + 1];
  if (b <= a) return;  // no stage: written by the attention kernel
  auto cta_of = [&](long long s) { return (int)(((s + 1) * P - 1) / T); };
  auto cta_start = [&](int c) { return (T * c) / P; };
  const int ca = cta_of(a), cb = cta_of(b - 1);
  if (ca == cb) return;  // one CTA did the whole unit and wrote it
  const int r = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const UnitCoord uc = unit_coord(p, u);
  const int t = r >> 7, sub = (r >> 6) & 1;
  const int tl = uc.qs * 64 + (r & 63);
  const int tok = uc.d.q_start + tl;
  const int hl_raw = uc.hh * p.HPU + 2 * t + sub;
  if (!((2 * t + sub) < p.HPU && hl_raw < p.G && tl < uc.d.L)) return;
  const int head = uc.g * p.G + hl_raw;
  auto slot_of = [&](int c) { return (c == ca && cta_start(c) < a) ? 2 * c + 1 : 2 * c; };
  float m = -INFINITY;
  for (int c = ca; c <= cb; ++c) m = fmaxf(m, p.LSEsk[(size_t)slot_of(c) * (NT * 128) + r]);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float tot = 0.f;
  if (m != -INFINITY) {
    for (int c = ca; c <= cb; ++c) {
      const int sl = slot_of(c);
      const float ls = p.LSEsk[(size_t)sl * (NT * 128) + r];
      if (ls == -INFINITY) continue;
      const float w = __expf(ls - m);
      tot += w;
      const float* src = p.Osk + ((size_t)sl * (NT * 128) + r) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] += w * src[i];
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  const size_t o = ((size_t)tok * p.Hq + head) * D + lane * PER;
  if (p.out_f32) {
#pragma unroll
    for (int i = 0; i < PER; ++i) reinterpret_cast<float*>(p.O)[o + i] = acc[i] * inv;
  } else {
#pragma unroll
    for (int i = 0; i < PER; i += 2)
      *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(p.O) + o + i) =
          pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
  }
  if (lane == 0) p.LSE[(size_t)head * p.L + tok] = tot > 0.f ? m + __logf(tot) : -INFINITY;
}

// Merge the fp32 partials of a KV-range split by their LSE.
// One warp per (token, head) row; lane handles D/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256)
    split_combine_kernel(const float* __restrict__ Opart, const float* __restrict__ LSEpart,
                         int n_splits, int L, int Hq, void* O, float* LSE, int out_f32) {
  const int rowid = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (rowid >= L * Hq) return;
  const int tok = rowid / Hq, head = rowid % Hq;
  float m = -INFINITY;
  for (int s = 0; s < n_splits; ++s) m = fmaxf(m, LSEpart[((size_t)s * Hq + head) * L + tok]);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float tot = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < n_splits; ++s) {
      const float ls = LSEpart[((size_t)s * Hq + head) * L + tok];
      if (ls == -INFINITY) continue;
      const float w = __expf(ls - m);
      tot += w;
      const float* src = Opart + (((size_t)s * L + tok) * Hq + head) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] += w * src[i];
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  const size_t o = ((size_t)tok * Hq + head) * D + lane * PER;
  if (out_f32) {
#pragma unroll
    for (int i = 0; i < PER; ++i) reinterpret_cast<float*>(O)[o + i] = acc[i] * inv;
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) reinterpret_cast<__nv_bfloat16*>(O)[o + i] = __float2bfloat16_rn(acc[i] * inv);
  }
  if (lane == 0) LSE[(size_t)head * L + tok] = tot > 0.f ? m + __logf(tot) : -INFINITY;
}

// fp32 -> bf16 (round to nearest even), grid-stride, 4 elements per step.
__global__ void cast_f32_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                     size_t n) {
  const size_t n4 = n / 4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(src)[i];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(dst)[i] = o;
  }
  for (size_t i = n4 * 4 + blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// fp32 -> two bf16 terms: hi = rn(x), lo = rn(x - hi); hi + lo carries ~16
// significant bits of x.
__global__ void split_f32_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ hi,
                                      __nv_bfloat16* __restrict__ lo, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float x = src[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

// Batched calls: per-sequence descriptors and unit offsets from the caller's
// device arrays (one CTA, block-wide scan in chunks of blockDim.x sequences).
// A sequence whose offsets are inconsistent gets no work units and flags
// CA_FLAG_BOUNDS.
__global__ void __launch_bounds__(1024)
    varlen_setup_kernel(const int32_t* __restrict__ cu_q, const int32_t* __restrict__ prefix_len,
                        const int32_t* __restrict__ cu_pages, int num_seqs, int total_q, int B,
                        int Hkv, int nhalves, SeqDesc* __restrict__ out, int32_t* n_units,
                        int32_t* err) {
  __shared__ int warp_sum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < num_seqs; base += blockDim.x) {
    const int s = base + tid;
    SeqDesc d = {0, 0, 0, 0, 0, 0, 0, s};
    int units = 0;
    if (s < num_seqs) {
      const int q0 = cu_q[s], q1 = cu_q[s + 1], P = prefix_len[s];
      const int p0 = cu_pages[s], p1 = cu_pages[s + 1];
      const long long L = (long long)q1 - q0;
      const long long nK = (P + L + B - 1) / B;
      const bool ok = q0 >= 0 && q1 <= total_q && L >= 0 && P >= 0 && p0 >= 0 &&
                      (long long)p1 - p0 >= nK && P + L <= 0x7fffffffLL;
      if (ok) {
        d.q_start = q0;
        d.L = (int)L;
        d.P = P;
        d.nKblk = (int)nK;
        d.pt_off = p0;
        d.nqs = (int)((L + 63) / 64);
        units = d.nqs * Hkv * nhalves;
      } else {
        set_flag(err, CA_FLAG_BOUNDS);
      }
    }
    int incl = units;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    d.unit_start = before + incl - units;
    if (s < num_seqs) out[s] = d;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < nw; ++w) tot += warp_sum[w];
      carry += tot;
    }
    __syncthreads();
  }
  if (tid == 0) *n_units = carry;
}

// bf16 -> f16 (exact for |x| in [2^-14, 65504]; smaller values round as f16
// subnormals), for Q of the E4M3 path.
__global__ void cast_bf16_f16_kernel(const __nv_bfloat16* __restrict__ src,
                                     __half* __restrict__ dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2half_rn(__bfloat162float(src[i]));
}

// escale[g * nKblk + e] = 256 * (K_scale, V_scale) of the page behind table
// entry e of group g (entries past counts[g] are left as they are).
__global__ void gather_scales_kernel(const int32_t* __restrict__ tables,
                                     const int32_t* __restrict__ counts,
                                     const int32_t* __restrict__ page_table,
                                     const float* __restrict__ K_scale,
                                     const float* __restrict__ V_scale, int Hkv, int nKblk,
                                     int num_pages, float2* __restrict__ escale, int32_t* err) {
  const int g = blockIdx.y;
  const int cnt = min(max(counts[g], 0), nKblk);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < cnt; e += gridDim.x * blockDim.x) {
    int kb = tables[(size_t)g * nKblk + e];
    if (kb < 0 || kb >= nKblk) {
      set_flag(err, CA_FLAG_BOUNDS);
      kb = 0;
    }
    int pg = page_table[kb];
    if (pg < 0 || pg >= num_pages) {
      set_flag(err, CA_FLAG_BOUNDS);
      pg = 0;
    }
    // x 256: the widened f16 operands hold decode(byte) / 256
    escale[(size_t)g * nKblk + e] = make_float2(K_scale[(size_t)pg * Hkv + g] * 256.f,
                                                V_scale[(size_t)pg * Hkv + g] * 256.f);
  }
}

// One CTA waits on a barrier nobody arrives on, for at most limit_ns.
__global__ void wait_probe_kernel(int32_t* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(b, 0, limit_ns)) set_flag(err, CA_FLAG_TIMEOUT);
}

}  // namespace ca

namespace ca {

template <int D, int NT, bool QS, bool KV8>
static cudaError_t launch_attn_t(const CUtensorMap& q, const CUtensorMap& qlo,
                                 const CUtensorMap& k, const CUtensorMap& v, const AttnParams& p,
                                 int grid, cudaStream_t st) {
  using S = Smem<D, NT, QS, KV8>;
  static_assert(S::kAlloc <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(chunk_attn_kernel<D, NT, QS, KV8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
  if (e != cudaSuccess) return e;
  chunk_attn_kernel<D, NT, QS, KV8><<<grid, 128 + NT * 128, S::kAlloc, st>>>(q, qlo, k, v, p);
  return cudaGetLastError();
}

cudaError_t launch_chunk_attention(const CUtensorMap& q, const CUtensorMap& qlo,
                                   const CUtensorMap& k, const CUtensorMap& v,
                                   const AttnParams& p, int D, int NT, bool qsplit, bool kv8,
                                   int grid, cudaStream_t st) {
#define CA_LAUNCH(d_, nt_, qs_, kv8_)                                            \
  if (D == d_ && NT == nt_ && qsplit == qs_ && kv8 == kv8_)                      \
    return launch_attn_t<d_, nt_, qs_, kv8_>(q, qlo, k, v, p, grid, st);
  CA_LAUNCH(128, 2, false, false)
  CA_LAUNCH(128, 1, false, false)
  CA_LAUNCH(64, 2, false, false)
  CA_LAUNCH(64, 1, false, false)
  CA_LAUNCH(128, 2, true, false)
  CA_LAUNCH(128, 1, true, false)
  CA_LAUNCH(64, 2, true, false)
  CA_LAUNCH(64, 1, true, false)
  CA_LAUNCH(128, 2, false, true)
  CA_LAUNCH(128, 1, false, true)
  CA_LAUNCH(64, 2, false, true)
  CA_LAUNCH(64, 1, false, true)
#undef CA_LAUNCH
  return cudaErrorInvalidValue;
}

cudaError_t launch_sk_combine(const AttnParams& p, int D, int NT, cudaStream_t st) {
  const dim3 grid(p.n_units, NT * 128 / 8);
  if (D == 128 && NT == 2) sk_combine_kernel<128, 2><<<grid, 256, 0, st>>>(p);
  else if (D == 128 && NT == 1) sk_combine_kernel<128, 1><<<grid, 256, 0, st>>>(p);
  else if (D == 64 && NT == 2) sk_combine_kernel<64, 2><<<grid, 256, 0, st>>>(p);
  else if (D == 64 && NT == 1) sk_combine_kernel<64, 1><<<grid, 256, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_split_combine(const float* Opart, const float* LSEpart, int n_splits, int L,
                                 int Hq, int D, void* O, float* LSE, int out_f32,
                                 cudaStream_t st) {
  const int rows = L * Hq;
  const int grid = (rows + 7) / 8;
  if (D == 128)
    split_combine_kernel<128><<<grid, 256, 0, st>>>(Opart, LSEpart, n_splits, L, Hq, O, LSE, out_f32);
  else if (D == 64)
    split_combine_kernel<64><<<grid, 256, 0, st>>>(Opart, LSEpart, n_splits, L, Hq, O, LSE, out_f32);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_cast_f32_bf16(const float* src, void* dst, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n / 4 + 255) / 256;
  if (blocks > (size_t)num_sms() * 16) blocks = (size_t)num_sms() * 16;
  if (blocks < 1) blocks = 1;
  cast_f32_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, reinterpret_cast<__nv_bfloat16*>(dst), n);
  return cudaGetLastError();
}

cudaError_t launch_split_f32_bf16(const float* src, void* hi, void* lo, size_t n,
                                  cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > (size_t)num_sms() * 16) blocks = (size_t)num_sms() * 16;
  split_f32_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      src, reinterpret_cast<__nv_bfloat16*>(hi), reinterpret_cast<__nv_bfloat16*>(lo), n);
  return cudaGetLastError();
}

cudaError_t launch_varlen_setup(const int32_t* cu_q, const int32_t* prefix_len,
                                const int32_t* cu_pages, int num_seqs, int total_q, int B, int Hkv,
                                int nhalves, SeqDesc* out, int32_t* n_units, int32_t* err,
                                cudaStream_t st) {
  varlen_setup_kernel<<<1, 1024, 0, st>>>(cu_q, prefix_len, cu_pages, num_seqs, total_q, B, Hkv,
                                          nhalves, out, n_units, err);
  return cudaGetLastError();
}

cudaError_t launch_cast_bf16_f16(const void* src, void* dst, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > (size_t)num_sms() * 16) blocks = (size_t)num_sms() * 16;
  cast_bf16_f16_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(src), static_cast<__half*>(dst), n);
  return cudaGetLastError();
}

cudaError_t launch_gather_scales(const int32_t* tables, const int32_t* counts,
                                 const int32_t* page_table, const float* K_scale,
                                 const float* V_scale, int Hkv, int nKblk, int num_pages,
                                 float2* escale, int32_t* err, cudaStream_t st) {
  const dim3 grid((nKblk + 255) / 256, Hkv);
  gather_scales_kernel<<<grid, 256, 0, st>>>(tables, counts, page_table, K_scale, V_scale, Hkv,
                                             nKblk, num_pages, escale, err);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(int32_t* err, unsigned long long limit_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace ca
