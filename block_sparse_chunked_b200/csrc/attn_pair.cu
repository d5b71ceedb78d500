// attn_pair.cu — chunked-prefill attention over the selected KV blocks of a
// paged cache on CTA pairs: one tcgen05 MMA of M = 256 (cta_group::2) spans two
// SMs, with the score tile triple-buffered in TMEM (sm_100a, head_dim 128).
//
// "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection", Abstract: every query of a GQA group reads exactly the KV blocks
// of its group's table, in place in the paged cache, with no KV compaction.
//
// A pair of CTAs (a cluster of two, on two SMs) takes two work units of the
// same group and 64-token query span: CTA r holds the rows of head pair r of
// the group (64 tokens x 2 heads = 128 rows), so the pair covers 256 rows that
// share one table and therefore one stream of K/V pages.  Each 128-key stage
// is split between the two CTAs' shared memory: CTA r holds keys
// [64 r, 64 r + 64) of K (its page of the stage) and head-dim columns
// [64 r, 64 r + 64) of V for all 128 keys.  The even CTA's MMA warp issues
// S = Q K^T (M 256, N 128 keys) and O += P V (M 256, N 128 head-dim columns, P
// from each CTA's TMEM) for both; each CTA's tensor core computes its own 128
// rows.  So every page byte crosses from L2 into one SM only, half of what a
// one-SM tile of the same rows would need, while the score tile still has
// three TMEM buffers (S(j+3) issued right after PV(j)) and the softmax of each
// CTA runs back to back on its own rows.
//
// Synchronisation of the pair: the K/V/Q loads of both CTAs complete on the
// even CTA's barriers (tx bytes); MMA completion (tcgen05.commit with the
// pair mask) arrives on the barrier at the same offset in both CTAs; the
// softmax warps of both CTAs arrive on the even CTA's P-ready barriers
// (after tcgen05.fence::before_thread_sync, which orders their TMEM writes).  A stage whose table run has one 64-token page
// left gives the odd CTA a copy of that page: its keys are masked out and its
// P is never read (the PV MMA then runs over 64 keys only).
//
// Roles per CTA (352 threads, one CTA per SM): warps 0-7 softmax, warp 8 K
// loads (+ set-up), warp 9 TMEM allocation (both CTAs) and MMA issue (even
// CTA), warp 10 V loads.  Softmax warp w reads TMEM lanes 32 (w mod 4) ..
// + 31 (the rows of its sub-partition) and owns keys [64 h, 64 h + 64) of
// each stage, h = w / 4: two warps share each row, so every sub-partition
// has two independent instruction streams feeding its exponential unit.  The
// two halves of a row exchange their maxima (and at the end their sums)
// through shared memory, synchronised by an mbarrier of the sub-partition's
// 64 threads.  Every wait is bounded; on expiry the CTA sets CA_FLAG_TIMEOUT
// and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_common.cuh"
#include "compactattn.h"
#include "internal.h"
#include "ptx.cuh"

namespace ca {

namespace {

constexpr int kPStageKeys = 128;
constexpr int kPSBufs = 3;  // S / P buffers in TMEM
constexpr int kPNK = 4;     // K ring slots (this CTA's 64 keys of a stage)
constexpr int kPNV = 4;     // V ring slots (this CTA's 64 head-dim columns of a stage)
constexpr int kPThreads = 352;
constexpr int kPSoftmaxWarps = 8;

struct PairSmem {  // head_dim 128
  static constexpr int kQChunk = 128 * 128;    // Q: 128 rows x 128 B per 64 columns
  static constexpr int kQ = 2 * kQChunk;
  static constexpr int kKChunk = 64 * 128;     // K: 64 keys x 128 B per 64 columns
  static constexpr int kKSlot = 2 * kKChunk;
  static constexpr int kVSlot = 128 * 128;     // V: 128 keys x 64 columns
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQ;
  static constexpr int kVOff = kKOff + kPNK * kKSlot;
  static constexpr int kBarOff = kVOff + kPNV * kVSlot;
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[3],
  // p_full[3], pv_done[0], o_done, drain, xchg[4], pv_done[1]
  static constexpr int kNumBars = 1 + 2 * kPNK + 2 * kPNV + 2 * kPSBufs + 3 + 4 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // row maxima of the two key halves, by stage parity [2][2][128], and the
  // final row sums [2][128]
  static constexpr int kXMaxOff = kMiscOff + 64;
  static constexpr int kXSumOff = kXMaxOff + 2 * 2 * 128 * 4;
  // fused mode: the group's table built in the CTA (entries, union bits, count)
  static constexpr int kFentOff = kXSumOff + 2 * 128 * 4;
  static constexpr int kBytes = kFentOff + (kMaxFusedWords * 32 + kMaxFusedWords + 1) * 4;
  static constexpr int kAlloc = kBytes + 1024;
};

struct PairPiece {
  int u, split, nsplit, out, slot;
};

// Blocks 2q and 2q + 1 form cluster q.  Both CTAs of a pair get the same
// split of the two units of one (group, span): units 2 m and 2 m + 1.
__device__ __forceinline__ PairPiece pair_piece(const AttnParams& p, int rank) {
  PairPiece t;
  const int b = blockIdx.x, q = b >> 1;
  if (p.n_splits > 1) {
    const int m = q / p.n_splits;
    t.split = q % p.n_splits;
    t.u = 2 * m + rank;
    t.nsplit = p.n_splits;
    t.out = kOutSplit;
    t.slot = t.split;
  } else if (p.tail_k > 1 && b >= p.tail_start) {
    const int rq = (b - p.tail_start) >> 1;
    const int m = rq / p.tail_k;
    t.split = rq % p.tail_k;
    t.u = p.tail_start + 2 * m + rank;
    t.nsplit = p.tail_k;
    t.out = kOutTail;
    t.slot = (t.u - p.tail_start) * p.tail_k + t.split;
  } else {
    t.u = b;
    t.split = 0;
    t.nsplit = 1;
    t.out = kOutFinal;
    t.slot = 0;
  }
  return t;
}

}  // namespace

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    chunk_attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  static_assert(D == 128, "the pair kernel splits head_dim 128 into two 64-column halves");
  using S = PairSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bars = sbase + S::kBarOff;
  const uint32_t q_full = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + kPNK + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * kPNK + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 2 * kPNK + kPNV + s); };
  auto s_full = [&](int b) { return bars + 8u * (1 + 2 * kPNK + 2 * kPNV + b); };
  auto p_full = [&](int b) { return bars + 8u * (1 + 2 * kPNK + 2 * kPNV + kPSBufs + b); };
  const uint32_t pv0 = bars + 8u * (1 + 2 * kPNK + 2 * kPNV + 2 * kPSBufs);
  const uint32_t o_done = pv0 + 8u;
  const uint32_t drain = pv0 + 16u;
  auto xchg = [&](int q) { return pv0 + 24u + 8u * q; };  // halves of a sub-partition's rows
  // PV(j) completes on pv_done(j % 2).  When the softmax sees S(j) complete,
  // PV(j-3) has completed too (S(j) was issued after it), so a parity wait for
  // PV(j-1) on pv_done((j-1) % 2) cannot alias; the softmax waits only at
  // stages that rescale O.
  auto pv_done = [&](int j) { return j % 2 == 0 ? pv0 : pv0 + 56u; };
  int* misc = reinterpret_cast<int*>(sm + S::kMiscOff);
  // misc[0] tmem base, [1] live entries, [2] first stage, [3] end stage, [5] abort
  volatile int* abort_flag = misc + 5;

  const int rank = (int)cluster_ctarank();
  const bool leader = rank == 0;
  const PairPiece tp = pair_piece(p, rank);
  // A batched call's grid bounds its units; the unit count is even (two head
  // pairs per span), so both CTAs of a pair leave together, before any
  // barrier, cluster barrier or TMEM use.
  if (p.n_units_dev && tp.u - rank >= *p.n_units_dev) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int spb = kPStageKeys / p.B;  // pages per stage
  const UnitCoord uc = unit_coord(p, tp.u);

  int32_t* fent = reinterpret_cast<int32_t*>(sm + S::kFentOff);
  if (warp == 8) {
    if (lane == 0) {
      misc[5] = 0;
      mbar_init(q_full, 1);
      for (int s = 0; s < kPNK; ++s) {
        mbar_init(k_full(s), 1);
        mbar_init(k_empty(s), 1);
      }
      for (int s = 0; s < kPNV; ++s) {
        mbar_init(v_full(s), 1);
        mbar_init(v_empty(s), 1);
      }
      for (int b = 0; b < kPSBufs; ++b) {
        mbar_init(s_full(b), 1);
        mbar_init(p_full(b), 2 * kPSoftmaxWarps);  // every softmax warp of both CTAs
      }
      mbar_init(pv_done(0), 1);
      mbar_init(pv_done(1), 1);
      mbar_init(o_done, 1);
      mbar_init(drain, 1);
      for (int q = 0; q < 4; ++q) mbar_init(xchg(q), 2);
      fence_mbar_init();
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    if (!p.mask_bits) {
      const int live = unit_live_warp(p, uc);  // the same for both units of the pair
      if (lane == 0) {
        const int nst = (live + spb - 1) / spb;
        misc[1] = live;
        misc[2] = (int)((long long)tp.split * nst / tp.nsplit);
        misc[3] = (int)((long long)(tp.split + 1) * nst / tp.nsplit);
      }
    }
  } else if (warp == 9) {
    tmem_alloc_pair(sbase + S::kMiscOff, 512);
    tmem_relinquish_pair();
  }
  if (p.mask_bits) {
    // fused mode: the whole CTA builds its group's table from the bit-packed
    // masks (both CTAs of a pair build the same one); one CTA per group writes
    // it out
    const int cnt = fused_group_table(p, uc, fent, kPThreads);
    if (uc.qs == 0 && uc.hh == 0 && tp.split == 0) {
      if (p.tables_out) {
        int32_t* trow_out = p.tables_out + (size_t)uc.g * uc.d.nKblk;
        for (int e = threadIdx.x; e < uc.d.nKblk; e += kPThreads)
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
      const int nst = (lo + spb - 1) / spb;
      misc[1] = lo;
      misc[2] = (int)((long long)tp.split * nst / tp.nsplit);
      misc[3] = (int)((long long)(tp.split + 1) * nst / tp.nsplit);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or commit targets them
  tc_fence_after();
  const uint32_t tmem = (uint32_t)misc[0];
  const int live = misc[1], s0 = misc[2], s1 = misc[3];
  const int n = s1 - s0;  // stages of this piece (equal in both CTAs)

  if (warp == 8 || warp == 10) {
    // ================================================================ loads
    // Warp 8: this CTA's Q rows (once) and its half of each K stage; warp 10:
    // its half of each V stage.  Copies complete on the even CTA's barriers;
    // the even CTA's warps announce the bytes of both halves.  Lane i looks
    // up table entry (base + i) and its page, 32 at a time.
    const bool is_k = warp == 8;
    const int nslots = is_k ? kPNK : kPNV;
    const uint32_t ring = sbase + (is_k ? S::kKOff : S::kVOff);
    const int slot_bytes = is_k ? S::kKSlot : S::kVSlot;
    const CUtensorMap* tm = is_k ? &tmK : &tmV;
    const uint64_t pol = policy_evict_last();
    if (is_k) {
      const uint32_t qf = mapa_rank(q_full, 0);
      if (leader && lane == 0) mbar_expect_tx(q_full, 2 * 128 * D * 2);
      if (lane == 0) {
        const uint64_t qpol = policy_evict_first();
        for (int s = 0; s < 2; ++s) {
          const int hl = min(p.G - 1, uc.hh * 2 + s);  // head within the group
          const int head = uc.g * p.G + hl;
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(sbase + S::kQOff + c * S::kQChunk + s * 64 * 128, &tmQ, qf, c * 64,
                             head, uc.d.q_start + uc.qs * 64, qpol);
        }
      }
    }
    const int32_t* trow = p.mask_bits ? fent : table_row(p, uc);
    const int e_begin = s0 * spb, e_end = min(live, s1 * spb);
    int pg_cache = 0, cache_base = -64;
    bool ok = true;
    auto page_of = [&](int e) {  // warp-wide: the physical page of table entry e
      if (e >= cache_base + 32) {
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
      return __shfl_sync(0xffffffffu, pg_cache, e - cache_base);
    };
    for (int j = 0; j < n && ok; ++j) {
      const int stage = s0 + j, slot = j % nslots, round = j / nslots;
      const uint32_t full = is_k ? k_full(slot) : v_full(slot);
      const uint32_t empty = is_k ? k_empty(slot) : v_empty(slot);
      const int npg = min(spb, live - stage * spb);
      // pages of the stage: K needs one (this CTA's keys), V all of them
      int page[2] = {0, 0};
      if (is_k) {
        const int pi = (spb == 2 && npg == 2) ? rank : 0;  // a lone page: both CTAs load it
        page[0] = page_of(stage * spb + pi);
      } else {
        for (int pi = 0; pi < npg; ++pi) page[pi] = page_of(stage * spb + pi);
      }
      if (round > 0) ok = wait_warp(empty, (round - 1) & 1, p, abort_flag);
      if (!ok) break;
      const uint32_t half = is_k ? (uint32_t)S::kKSlot : (uint32_t)npg * p.B * 128;
      if (leader) mbar_expect_tx_w(full, 2 * half);
      const uint32_t full_cl = mapa_rank(full, 0);
      const uint32_t dst = ring + slot * slot_bytes;
      if (is_k) {
        const int row0 = spb == 1 ? 64 * rank : 0;  // 128-token pages: this CTA's 64 rows
        for (int c = 0; c < 2; ++c)
          tma_load_4d_pair_w(dst + c * S::kKChunk, tm, full_cl, c * 64, row0, uc.g, page[0], pol);
      } else {
        for (int pi = 0; pi < npg; ++pi)
          tma_load_4d_pair_w(dst + pi * p.B * 128, tm, full_cl, 64 * rank, 0, uc.g, page[pi], pol);
      }
    }
    if (leader && lane == 0) {
      // Do not leave with copies in flight (both CTAs' copies complete here;
      // the odd CTA stays resident until the pair's closing cluster barrier).
      for (int j = max(0, n - nslots); j < n; ++j)
        mbar_wait(is_k ? k_full(j % nslots) : v_full(j % nslots), (j / nslots) & 1, p.wait_ns);
      if (is_k) mbar_wait(q_full, 0, p.wait_ns);
    }
  } else if (warp == 9) {
    // ================================================================ MMA issuer (even CTA)
    if (leader) {
      constexpr uint32_t kIdescS = idesc_bf16(256, 128, 0);
      constexpr uint32_t kIdescPV = idesc_bf16(256, D, 1);
      const uint64_t qdesc = smem_desc_sw128(sbase + S::kQOff, 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(sbase + S::kKOff, 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(sbase + S::kVOff, S::kVSlot, 1024);
      auto keys_of = [&](int j) { return min(spb, live - (s0 + j) * spb) * p.B; };
      auto issue_s = [&](int j) {  // N = 128 keys: 64 from each CTA
        const uint64_t kd = kdesc0 + (uint64_t)(((j % kPNK) * S::kKSlot) >> 4);
        const uint32_t dt = tmem + 128 + (j % kPSBufs) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = ((kk >> 2) * S::kQChunk + (kk & 3) * 32) >> 4;
          const uint32_t offk = ((kk >> 2) * S::kKChunk + (kk & 3) * 32) >> 4;
          mma_ss_pair_w(dt, qdesc + offq, kd + offk, kIdescS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int j) {  // N = 128 head-dim columns: 64 from each CTA
        const uint64_t vd = vdesc0 + (uint64_t)(((j % kPNV) * S::kVSlot) >> 4);
        const uint32_t at = tmem + 128 + (j % kPSBufs) * 128;
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        const int nk = keys_of(j) / 16;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          if (kk < nk)
            mma_ts_pair_w(tmem, at + (kk & 3) * 8 + (kk >> 2) * 64,
                          vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV,
                          kk > 0 ? 1u : acc0);
      };
      bool ok = true;
      if (n > 0) {
        ok = wait_warp(q_full, 0, p, abort_flag);
        for (int j = 0; j < min(kPSBufs, n) && ok; ++j) {
          ok = wait_warp(k_full(j % kPNK), (j / kPNK) & 1, p, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(j);
          mma_commit_pair_w(s_full(j % kPSBufs));
          mma_commit_pair_w(k_empty(j % kPNK));
        }
        for (int j = 0; j < n && ok; ++j) {
          const int b = j % kPSBufs;
          ok = wait_warp(p_full(b), (j / kPSBufs) & 1, p, abort_flag) &&
               wait_warp(v_full(j % kPNV), (j / kPNV) & 1, p, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j);
          mma_commit_pair_w(v_empty(j % kPNV));
          mma_commit_pair_w(pv_done(j));
          const int jn = j + kPSBufs;
          if (jn < n) {
            // S(j+3) reuses buffer b after PV(j) has read P(j) (in-order MMAs)
            ok = wait_warp(k_full(jn % kPNK), (jn / kPNK) & 1, p, abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_s(jn);
            mma_commit_pair_w(s_full(b));
            mma_commit_pair_w(k_empty(jn % kPNK));
          }
        }
        if (ok) mma_commit_pair_w(o_done);
      }
      mma_commit_pair_w(drain);  // arrives in both CTAs once every MMA has finished
    }
    mbar_wait(drain, 0, p.wait_ns);
  } else {
    // ================================================================ softmax / epilogue
    const int q4 = warp & 3;          // TMEM lane quadrant (sub-partition)
    const int h = warp >> 2;          // key half of each stage: [64 h, 64 h + 64)
    const int row = q4 * 32 + lane;   // 0..127 = TMEM lane
    const int sub = row >> 6;         // head of the pair
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + lane_off + 64 * h;  // this warp's 64 columns of O
    float* xmax = reinterpret_cast<float*>(sm + S::kXMaxOff);  // [2][2][128]
    float* xsum = reinterpret_cast<float*>(sm + S::kXSumOff);  // [2][128]
    const int t0 = uc.qs * 64;
    const int tl = t0 + (row & 63);
    const int tok = uc.d.q_start + tl;
    const int hl_raw = uc.hh * 2 + sub;
    const bool valid_row = hl_raw < p.G && tl < uc.d.L;
    const int head = uc.g * p.G + min(hl_raw, p.G - 1);
    const int32_t* trow = p.mask_bits ? fent : table_row(p, uc);
    const int kb_m0 = (uc.d.P + t0) / p.B;
    int mask_e = live;
    while (mask_e > 0 && trow[mask_e - 1] >= kb_m0) --mask_e;
    const int kposA = mask_e < live ? trow[mask_e] * p.B : 0;
    const int kposB = kposA + p.B;
    const int qpos = uc.d.P + tl;
    constexpr int kHalf = kPStageKeys / 2;
    float m_used = -INFINITY, l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int stage = s0 + j, b = j % kPSBufs;
      const int npg = min(spb, live - stage * spb);
      const int nvalid = npg * p.B;
      const bool mine = h * kHalf < nvalid;  // this half holds keys of the stage (warp-uniform)
      const bool mask_stage = stage * spb + npg > mask_e;
      const uint32_t tS = tmem + lane_off + 128 + b * 128;
      ok = wait_warp(s_full(b), (j / kPSBufs) & 1, p, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float sr[kHalf];
      if (mine) {
        tmem_ld64f(tS + h * kHalf, sr);
        tmem_wait_ld();
        if (mask_stage) {  // keys after this row's position -> -inf
          const int e0 = stage * spb;
          const int pm = max(0, mask_e - e0);
          const int cm0 = pm * p.B;
          const int lim = qpos - (e0 + pm > mask_e ? kposB : kposA);
#pragma unroll
          for (int c = 0; c < kHalf; ++c) {
            const int cc = h * kHalf + c;
            if (cc >= cm0 && (cc - cm0) > lim) sr[c] = -INFINITY;
          }
        }
      }
      // exponentiate this half against the running max; P (bf16 pairs) goes
      // to TMEM columns [64 h, 64 h + 32) of the buffer: inside this warp's
      // own half of S, which the other warp of the row never reads (PV takes
      // keys 64 .. 127 from column 64)
      const float sc = p.scale_log2;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      auto pass = [&](float nm) {
        a0 = a1 = a2 = a3 = 0.f;
#pragma unroll
        for (int c = 0; c < kHalf / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            ffma2(x0, x1, sr[c * 32 + 2 * i], sr[c * 32 + 2 * i + 1], sc, sc, nm, nm);
            const float e0 = ex2(x0), e1 = ex2(x1);
            if (i & 1) fadd2(a2, a3, e0, e1);
            else fadd2(a0, a1, e0, e1);
            pk[i] = pack_bf16x2(e0, e1);
          }
          tmem_st16(tS + h * kHalf + c * 16, pk);
        }
      };
      // The max of the half is needed only if it may exceed m_used + 8, i.e.
      // if some exponential exceeds 2^8: never while the sum of the half's
      // (positive) exponentials stays <= 256, and always before the row has
      // a max.  Otherwise the half cannot move the max and reports -inf.
      float pmax = -INFINITY;
      if (mine) {
        pass(m_used == -INFINITY ? 0.f : -m_used);
        const float asum = (a0 + a1) + (a2 + a3);
        const bool big = !(asum <= 256.f) || m_used == -INFINITY;
        if (__any_sync(0xffffffffu, big)) {
          float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int i = 0; i < kHalf / 2; ++i) {
            if (i & 1) mx1 = max3(mx1, sr[2 * i], sr[2 * i + 1]);
            else mx0 = max3(mx0, sr[2 * i], sr[2 * i + 1]);
          }
          pmax = fmaxf(mx0, mx1);
        }
      }
      // the row's max: both halves, through shared memory (slots alternate by
      // stage, so a fast warp never overwrites a value its partner still reads)
      float* xm = xmax + (j & 1) * 256;
      xm[h * 128 + row] = pmax;
      __syncwarp();
      if (lane == 0) mbar_arrive(xchg(q4));  // one phase per stage: one arrival per warp
      ok = wait_warp(xchg(q4), j & 1, p, abort_flag);
      if (!ok) break;
      const float mx = fmaxf(pmax, xm[(1 - h) * 128 + row]) * sc;
      const float m_new = fmaxf(m_used, mx);
      const bool need = (m_new != -INFINITY) && (m_new > m_used + 8.0f);
      float alpha = 1.f;
      const bool redo = __any_sync(0xffffffffu, need);
      if (redo) {  // both halves decide alike
        if (need) {
          alpha = ex2(m_used - m_new);
          l0 *= alpha;
          l1 *= alpha;
          l2 *= alpha;
          l3 *= alpha;
          m_used = m_new;
        }
        if (mine) {
          tmem_wait_st();
          pass(m_used == -INFINITY ? 0.f : -m_used);
        }
      }
      l0 += a0;
      l1 += a1;
      l2 += a2;
      l3 += a3;
      if (j > 0 && redo) {
        // O holds the sum over earlier stages at the old max: PV(j-1) must
        // have finished before this warp's 64 columns of O are rescaled
        ok = wait_warp(pv_done(j - 1), ((j - 1) >> 1) & 1, p, abort_flag);
        if (!ok) break;
        {
          tc_fence_after();
          uint32_t r[32];
          for (int c = 0; c < 2; ++c) {
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_rank(p_full(b), 0));
    }
    // ---- epilogue: the row sum of both halves, then this warp's 64 columns
    const float lpart = (l0 + l1) + (l2 + l3);
    float l = lpart;
    if (ok) {
      xsum[h * 128 + row] = lpart;
      __syncwarp();
      if (lane == 0) mbar_arrive(xchg(q4));  // phase n
      ok = wait_warp(xchg(q4), n & 1, p, abort_flag);
      if (ok) l += xsum[(1 - h) * 128 + row];
    }
    const bool ran = ok && n > 0;
    bool have_o = false;
    if (ran) {
      have_o = wait_warp(o_done, 0, p, abort_flag);
      if (have_o) tc_fence_after();
    }
    const bool have = have_o && l > 0.f;
    const float inv = have ? 1.f / l : 0.f;
    const float lse = have ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    uint32_t r[32];
    for (int c = 0; c < 2; ++c) {
      if (have_o) {
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      if (!valid_row) continue;
      const int col = 64 * h + 32 * c;
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = have ? __uint_as_float(r[i]) * inv : 0.f;
      float* fdst = nullptr;
      if (tp.out == kOutSplit)
        fdst = p.Opart + (((size_t)tp.slot * p.L + tok) * p.Hq + head) * D + col;
      else if (tp.out == kOutTail)
        fdst = p.Otail + ((size_t)tp.slot * 128 + row) * D + col;
      if (fdst) {
        float4* dst = reinterpret_cast<float4*>(fdst);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.O) +
                                              ((size_t)tok * p.Hq + head) * D + col);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]),
                              pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                              pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                              pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
      }
    }
    if (valid_row && h == 0) {
      if (tp.out == kOutSplit) p.LSEpart[((size_t)tp.slot * p.Hq + head) * p.L + tok] = lse;
      else if (tp.out == kOutTail) p.LSEtail[(size_t)tp.slot * 128 + row] = lse;
      else p.LSE[(size_t)head * p.L + tok] = lse;
    }
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync_all();  // no MMA of the pair reads this CTA's memory any more
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

cudaError_t launch_chunk_attention_pair(const CUtensorMap& q, const CUtensorMap& k,
                                        const CUtensorMap& v, const AttnParams& p, int D,
                                        int grid, cudaStream_t st) {
  if (D != 128 || (grid & 1)) return cudaErrorInvalidValue;
  static_assert(PairSmem::kAlloc <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(chunk_attn_pair_kernel<128>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       PairSmem::kAlloc);
  if (e != cudaSuccess) return e;
  chunk_attn_pair_kernel<128><<<grid, kPThreads, PairSmem::kAlloc, st>>>(q, k, v, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.tail_k <= 1 || p.n_tail <= 0) return e;
  return launch_tail_combine(p, D, st);
}

}  // namespace ca
