// attn_tile.cu — chunked-prefill attention over the selected KV blocks of a
// paged cache, one 128-row tile per CTA with the score tile triple-buffered in
// tensor memory (sm_100a: tcgen05, TMEM, TMA).
//
// "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection", Abstract: every query of a GQA group reads exactly the KV blocks
// of its group's table, in place in the paged cache, with no KV compaction.
//
// Work unit = (KV group g, 64-token query span qs, head pair hh): the span's
// 64 tokens for two query heads of the group stacked into one M = 128 tile, so
// every K/V page fetched feeds one QK^T and one PV MMA of 128 rows.  The live
// blocks of a span are a prefix of the group's sorted table; only the last one
// or two (those past the span's first query position) need a token mask.
//
// Why three score buffers: with one, the score tile of stage j+1 can only be
// computed after the softmax of stage j has written P(j) and PV(j) has been
// issued, so every stage pays softmax -> handshake -> PV -> QK^T in series.
// Here S(j+3) is issued right after PV(j), so the softmax warps find the next
// score tile ready and run back to back, and the tensor pipe works on S(j+1..)
// and PV while they do.  TMEM columns: O [0, 128), S/P buffer b at
// 128 + 128 b (b = 0, 1, 2); P (bf16) overwrites the first 64 columns of its
// S buffer and is read by the PV MMA from there.
//
// Roles (224 threads, one CTA per SM):
//   warps 0-3  softmax: one thread per row; loads the row's 128 scores from
//              TMEM, applies the diagonal token mask, exponentiates against the
//              running max while it takes the new row max (the max is moved
//              only when it grows by more than 2^8, exact; then the stage is
//              redone against the new max), keeps the fp32 row sum, writes P as
//              bf16 back to TMEM; rescales O when the max moves; finally
//              normalises O and writes O / LSE (or partials);
//   warp 4     K producer: Q once, then K pages (3-slot ring) through tables ->
//              page_table -> physical page;
//   warp 5     TMEM allocator and tcgen05.mma issuer;
//   warp 6     V producer: V pages (2-slot ring).  K and V have producers of
//              their own so that each ring refills as soon as its own slot is
//              free: K runs up to three stages ahead of the MMAs, V two.
// Every pipeline wait is bounded; on expiry the CTA sets CA_FLAG_TIMEOUT and
// unwinds instead of hanging.
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

constexpr int kTStageKeys = 128;  // keys per stage (two 64-token pages or one 128-token page)
constexpr int kTSBufs = 3;        // S / P buffers in TMEM
constexpr int kTNK = 3;           // K ring slots
constexpr int kTNV = 2;           // V ring slots
constexpr int kTThreads = 224;

template <int D>
struct TileSmem {
  static constexpr int kChunkBytes = 128 * 128;           // 128 rows x 128 B (64 bf16)
  static constexpr int kQ = 128 * D * 2;                  // the Q tile
  static constexpr int kKV = kTStageKeys * D * 2;         // one stage of K (or V)
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQ;
  static constexpr int kVOff = kKOff + kTNK * kKV;
  static constexpr int kBarOff = kVOff + kTNV * kKV;
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[3],
  // p_full[3], pv_done[0], o_done, drain, pv_done[1]
  static constexpr int kNumBars = 1 + 2 * kTNK + 2 * kTNV + 2 * kTSBufs + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  static constexpr int kAlloc = kBytes + 1024;            // slack for 1024-byte alignment
};

// This CTA's piece of work: unit, KV stage range and where its result goes.
struct TilePiece {
  int u, split, nsplit, out, slot;
};

__device__ __forceinline__ TilePiece tile_piece(const AttnParams& p) {
  TilePiece t;
  const int b = blockIdx.x;
  if (p.n_splits > 1) {  // every unit in n_splits pieces
    t.u = b / p.n_splits;
    t.split = b % p.n_splits;
    t.nsplit = p.n_splits;
    t.out = kOutSplit;
    t.slot = t.split;
  } else if (p.tail_k > 1 && b >= p.tail_start) {  // the last partial wave, split
    const int r = b - p.tail_start;
    t.u = p.tail_start + r / p.tail_k;
    t.split = r % p.tail_k;
    t.nsplit = p.tail_k;
    t.out = kOutTail;
    t.slot = r;
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
__global__ void __launch_bounds__(kTThreads, 1)
    chunk_attn_tile_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using S = TileSmem<D>;
  constexpr int KCH = D / 64;  // 64-element (128-byte) chunks along head_dim
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bars = sbase + S::kBarOff;
  const uint32_t q_full = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + kTNK + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * kTNK + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 2 * kTNK + kTNV + s); };
  auto s_full = [&](int b) { return bars + 8u * (1 + 2 * kTNK + 2 * kTNV + b); };
  auto p_full = [&](int b) { return bars + 8u * (1 + 2 * kTNK + 2 * kTNV + kTSBufs + b); };
  const uint32_t pv0 = bars + 8u * (1 + 2 * kTNK + 2 * kTNV + 2 * kTSBufs);
  const uint32_t o_done = pv0 + 8u;
  const uint32_t drain = pv0 + 16u;
  // PV(j) completes on pv_done(j % 2).  When the softmax sees S(j) complete,
  // PV(j-3) has completed too (S(j) was issued after it), so a parity wait for
  // PV(j-1) on pv_done((j-1) % 2) cannot alias; the softmax waits only at
  // stages that rescale O.
  auto pv_done = [&](int j) { return j % 2 == 0 ? pv0 : pv0 + 24u; };
  int* misc = reinterpret_cast<int*>(sm + S::kMiscOff);
  // misc[0] tmem base, [1] live entries, [2] first stage, [3] end stage, [5] abort
  volatile int* abort_flag = misc + 5;

  // A batched call's grid is an upper bound on its units: surplus CTAs leave
  // before touching shared memory, barriers or TMEM.
  const TilePiece tp = tile_piece(p);
  if (p.n_units_dev && tp.u >= *p.n_units_dev) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int spb = kTStageKeys / p.B;  // pages per stage
  const UnitCoord uc = unit_coord(p, tp.u);

  if (warp == 4) {
    // barriers, then Q (it does not depend on the table), then the live prefix
    if (lane == 0) {
      misc[5] = 0;
      mbar_init(q_full, 1);
      for (int s = 0; s < kTNK; ++s) {
        mbar_init(k_full(s), 1);
        mbar_init(k_empty(s), 1);
      }
      for (int s = 0; s < kTNV; ++s) {
        mbar_init(v_full(s), 1);
        mbar_init(v_empty(s), 1);
      }
      for (int b = 0; b < kTSBufs; ++b) {
        mbar_init(s_full(b), 1);
        mbar_init(p_full(b), 4);  // one arrival per softmax warp
      }
      mbar_init(pv_done(0), 1);
      mbar_init(pv_done(1), 1);
      mbar_init(o_done, 1);
      mbar_init(drain, 1);
      fence_mbar_init();
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(q_full, 128 * D * 2);
      for (int s = 0; s < 2; ++s) {
        const int hl = min(p.G - 1, uc.hh * 2 + s);  // head within the group
        const int head = uc.g * p.G + hl;
        for (int c = 0; c < KCH; ++c)
          tma_load_3d(sbase + S::kQOff + c * S::kChunkBytes + s * 64 * 128, &tmQ, q_full, c * 64,
                      head, uc.d.q_start + uc.qs * 64);
      }
    }
    const int live = unit_live_warp(p, uc);
    if (lane == 0) {
      const int nst = (live + spb - 1) / spb;
      misc[1] = live;
      misc[2] = (int)((long long)tp.split * nst / tp.nsplit);
      misc[3] = (int)((long long)(tp.split + 1) * nst / tp.nsplit);
    }
  } else if (warp == 5) {
    tmem_alloc(sbase + S::kMiscOff, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)misc[0];
  const int live = misc[1], s0 = misc[2], s1 = misc[3];
  const int n = s1 - s0;  // stages of this piece

  if (warp == 4 || warp == 6) {
    // ================================================================ producers
    // The whole warp runs the loop: lane i looks up table entry (base + i) and
    // its page id, 32 at a time, so the dependent lookups tables -> page_table
    // are off the per-stage path; one elected lane issues the copies.  Warp 4
    // streams K pages, warp 6 V pages, each in stage order into its own ring.
    const bool is_k = warp == 4;
    const int nslots = is_k ? kTNK : kTNV;
    const uint32_t ring = sbase + (is_k ? S::kKOff : S::kVOff);
    const CUtensorMap* tm = is_k ? &tmK : &tmV;
    const uint64_t pol = policy_evict_last();
    const int32_t* trow = table_row(p, uc);
    const int e_begin = s0 * spb, e_end = min(live, s1 * spb);
    int pg_cache = 0, cache_base = -64;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int stage = s0 + j, slot = j % nslots, round = j / nslots;
      const uint32_t full = is_k ? k_full(slot) : v_full(slot);
      const uint32_t empty = is_k ? k_empty(slot) : v_empty(slot);
      const int npg = min(spb, live - stage * spb);
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
      if (round > 0) ok = wait_warp(empty, (round - 1) & 1, p, abort_flag);
      if (!ok) break;
      mbar_expect_tx_w(full, (uint32_t)npg * p.B * D * 2);
      for (int pi = 0; pi < npg; ++pi)
        for (int c = 0; c < KCH; ++c)
          tma_load_4d_w(ring + slot * S::kKV + c * S::kChunkBytes + pi * p.B * 128, tm, full,
                        c * 64, 0, uc.g, page[pi], pol);
    }
    if (lane == 0) {
      // Do not leave with copies in flight: the last stages' loads must land.
      for (int j = max(0, n - nslots); j < n; ++j)
        mbar_wait(is_k ? k_full(j % nslots) : v_full(j % nslots), (j / nslots) & 1, p.wait_ns);
      if (is_k) mbar_wait(q_full, 0, p.wait_ns);
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    // The whole warp runs this loop (addresses stay warp-uniform); one elected
    // lane issues each tcgen05.mma / commit.  Descriptors differ per MMA only
    // in the start-address field: built once, advanced by compile-time offsets.
    constexpr uint32_t kIdescPV = idesc_bf16(128, D, 1);
    constexpr uint32_t kIdescS128 = idesc_bf16(128, 128, 0);
    constexpr uint32_t kIdescS64 = idesc_bf16(128, 64, 0);
    const uint64_t qdesc = smem_desc_sw128(sbase + S::kQOff, 16, 1024);
    const uint64_t kdesc0 = smem_desc_sw128(sbase + S::kKOff, 16, 1024);
    const uint64_t vdesc0 = smem_desc_sw128(sbase + S::kVOff, S::kChunkBytes, 1024);
    auto keys_of = [&](int j) { return min(spb, live - (s0 + j) * spb) * p.B; };
    auto issue_s = [&](int j) {
      const uint64_t kd = kdesc0 + (uint64_t)(((j % kTNK) * S::kKV) >> 4);
      const uint32_t idesc = keys_of(j) == 128 ? kIdescS128 : kIdescS64;
      const uint32_t dt = tmem + 128 + (j % kTSBufs) * 128;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * S::kChunkBytes + (kk & 3) * 32) >> 4;
        mma_ss_w(dt, qdesc + off, kd + off, idesc, kk > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](int j) {
      const uint64_t vd = vdesc0 + (uint64_t)(((j % kTNV) * S::kKV) >> 4);
      const uint32_t at = tmem + 128 + (j % kTSBufs) * 128;
      const uint32_t acc0 = j > 0 ? 1u : 0u;
      if (keys_of(j) == 128) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_w(tmem, at + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV,
                   kk > 0 ? 1u : acc0);
      } else {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_w(tmem, at + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV,
                   kk > 0 ? 1u : acc0);
      }
    };
    bool ok = true;
    if (n > 0) {
      ok = wait_warp(q_full, 0, p, abort_flag);
      for (int j = 0; j < min(kTSBufs, n) && ok; ++j) {
        ok = wait_warp(k_full(j % kTNK), (j / kTNK) & 1, p, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_s(j);
        mma_commit_w(s_full(j % kTSBufs));
        mma_commit_w(k_empty(j % kTNK));
      }
      for (int j = 0; j < n && ok; ++j) {
        const int b = j % kTSBufs;
        ok = wait_warp(p_full(b), (j / kTSBufs) & 1, p, abort_flag) &&
             wait_warp(v_full(j % kTNV), (j / kTNV) & 1, p, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j);
        mma_commit_w(v_empty(j % kTNV));
        mma_commit_w(pv_done(j));
        const int jn = j + kTSBufs;
        if (jn < n) {
          // S(j+3) reuses buffer b: it runs after PV(j) has read P(j) (the
          // tensor pipe executes one thread's MMAs in issue order)
          ok = wait_warp(k_full(jn % kTNK), (jn / kTNK) & 1, p, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(jn);
          mma_commit_w(s_full(b));
          mma_commit_w(k_empty(jn % kTNK));
        }
      }
      if (ok) mma_commit_w(o_done);  // this piece's O is complete
    }
    // every MMA issued by this warp has finished before TMEM is released
    mma_commit_w(drain);
    mbar_wait(drain, 0, p.wait_ns);
  } else {
    // ================================================================ softmax / epilogue
    const int row = threadIdx.x;  // 0..127 = TMEM lane
    const int sub = row >> 6;     // head of the pair
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tmem + lane_off;
    const int t0 = uc.qs * 64;
    const int tl = t0 + (row & 63);     // token within the chunk
    const int tok = uc.d.q_start + tl;  // row of Q / O
    const int hl_raw = uc.hh * 2 + sub;
    const bool valid_row = hl_raw < p.G && tl < uc.d.L;
    const int head = uc.g * p.G + min(hl_raw, p.G - 1);
    const int32_t* trow = table_row(p, uc);
    // Token-level causal mask: only blocks that hold a key later than the
    // span's first query (kb >= (P + t0) / B) need it; in the ascending table
    // they are the last live entries, from mask_e on (at most two blocks).
    const int kb_m0 = (uc.d.P + t0) / p.B;
    int mask_e = live;
    while (mask_e > 0 && trow[mask_e - 1] >= kb_m0) --mask_e;
    const int kposA = mask_e < live ? trow[mask_e] * p.B : 0;
    const int kposB = kposA + p.B;
    const int qpos = uc.d.P + tl;  // this row's position: keys j <= qpos are visible
    float m_used = -INFINITY, l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int stage = s0 + j, b = j % kTSBufs;
      const int npg = min(spb, live - stage * spb);
      const int nvalid = npg * p.B;
      const bool mask_stage = stage * spb + npg > mask_e;
      const uint32_t tS = tmem + lane_off + 128 + b * 128;
      ok = wait_warp(s_full(b), (j / kTSBufs) & 1, p, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float sr[kTStageKeys];
      tmem_ld64f(tS, sr);
      if (nvalid > 64) tmem_ld64f(tS + 64, sr + 64);
      tmem_wait_ld();
      if (nvalid <= 64) {
#pragma unroll
        for (int c = 64; c < kTStageKeys; ++c) sr[c] = -INFINITY;
      }
      if (mask_stage) {  // keys after this row's position -> -inf
        const int e0 = stage * spb;
        const int pm = max(0, mask_e - e0);
        const int cm0 = pm * p.B;
        const int lim = qpos - (e0 + pm > mask_e ? kposB : kposA);  // visible while c - cm0 <= lim
#pragma unroll
        for (int c = 0; c < kTStageKeys; ++c)
          if (c >= cm0 && (c - cm0) > lim) sr[c] = -INFINITY;
      }
      // One pass over the row: p = 2^(s*scale - m) against the running max m
      // (packed FMA, then ex2; the fp32 sum is taken before the bf16 rounding),
      // P stored to TMEM chunk by chunk, and, independent of the exponentials,
      // the stage's row max of the raw scores (scale > 0 commutes with max).
      const float sc = p.scale_log2;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      auto pass = [&](float nm, bool with_max) {
        float mx0 = -INFINITY, mx1 = -INFINITY;
        a0 = a1 = a2 = a3 = 0.f;
#pragma unroll
        for (int c = 0; c < kTStageKeys / 32; ++c) {
          if (c * 32 < nvalid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float s0v = sr[c * 32 + 2 * i], s1v = sr[c * 32 + 2 * i + 1];
              if (with_max) {
                if (i & 1) mx1 = max3(mx1, s0v, s1v);
                else mx0 = max3(mx0, s0v, s1v);
              }
              float x0, x1;
              ffma2(x0, x1, s0v, s1v, sc, sc, nm, nm);
              const float e0 = ex2(x0), e1 = ex2(x1);
              if (i & 1) fadd2(a2, a3, e0, e1);  // two independent sum chains
              else fadd2(a0, a1, e0, e1);
              pk[i] = pack_bf16x2(e0, e1);
            }
            tmem_st16(tS + c * 16, pk);
          }
        }
        return fmaxf(mx0, mx1) * sc;
      };
      // Exponentiate against the running max first.  Only when the stage's max
      // exceeds it by more than 2^8 (always at the first stage, rarely later)
      // does the whole warp redo the stage against the new max: the TMEM
      // stores are warp-wide, and lanes whose max did not move recompute the
      // same values.
      const float mx = pass(m_used == -INFINITY ? 0.f : -m_used, true);
      const float m_new = fmaxf(m_used, mx);
      const bool need = (m_new != -INFINITY) && (m_new > m_used + 8.0f);
      float alpha = 1.f;
      const bool redo = __any_sync(0xffffffffu, need);
      if (redo) {
        if (need) {
          alpha = ex2(m_used - m_new);  // 0 when m_used == -inf
          l0 *= alpha;
          l1 *= alpha;
          l2 *= alpha;
          l3 *= alpha;
          m_used = m_new;
        }
        tmem_wait_st();  // the first pass's P stores complete before they are overwritten
        pass(m_used == -INFINITY ? 0.f : -m_used, false);
      }
      l0 += a0;
      l1 += a1;
      l2 += a2;
      l3 += a3;
      // O holds the sum over earlier stages at the old max: PV(j-1) must have
      // finished before O is rescaled
      if (j > 0 && redo) {
        ok = wait_warp(pv_done(j - 1), ((j - 1) >> 1) & 1, p, abort_flag);
        if (!ok) break;
        {
          tc_fence_after();
          uint32_t r[32];
          for (int c = 0; c < D / 32; ++c) {
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
      if (lane == 0) mbar_arrive(p_full(b));
    }
    // ---- epilogue
    const bool ran = ok && n > 0;
    bool have_o = false;
    if (ran) {
      have_o = wait_warp(o_done, 0, p, abort_flag);
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
      if (tp.out == kOutSplit)
        fdst = p.Opart + (((size_t)tp.slot * p.L + tok) * p.Hq + head) * D + c * 32;
      else if (tp.out == kOutTail)
        fdst = p.Otail + ((size_t)tp.slot * 128 + row) * D + c * 32;
      if (fdst) {
        float4* dst = reinterpret_cast<float4*>(fdst);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.O) +
                                              ((size_t)tok * p.Hq + head) * D + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]),
                              pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                              pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                              pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
      }
    }
    if (valid_row) {
      if (tp.out == kOutSplit) p.LSEpart[((size_t)tp.slot * p.Hq + head) * p.L + tok] = lse;
      else if (tp.out == kOutTail) p.LSEtail[(size_t)tp.slot * 128 + row] = lse;
      else p.LSE[(size_t)head * p.L + tok] = lse;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the pieces of the split tail units.  Block (t, r8) handles rows
// [8 r8, 8 r8 + 8) of tail unit t, one warp per row (lane = D/32 consecutive
// columns); piece k of unit t left its rows at Otail[t * tail_k + k].
template <int D>
__global__ void __launch_bounds__(256) tail_combine_kernel(const AttnParams p) {
  const int t = blockIdx.x;
  const int u = p.tail_start + t;
  const int r = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const UnitCoord uc = unit_coord(p, u);
  const int sub = r >> 6;
  const int tl = uc.qs * 64 + (r & 63);
  const int tok = uc.d.q_start + tl;
  const int hl_raw = uc.hh * 2 + sub;
  if (!(hl_raw < p.G && tl < uc.d.L)) return;
  const int head = uc.g * p.G + hl_raw;
  const int K = p.tail_k;
  float m = -INFINITY;
  for (int k = 0; k < K; ++k) m = fmaxf(m, p.LSEtail[((size_t)t * K + k) * 128 + r]);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float tot = 0.f;
  if (m != -INFINITY) {
    for (int k = 0; k < K; ++k) {
      const size_t sl = (size_t)t * K + k;
      const float ls = p.LSEtail[sl * 128 + r];
      if (ls == -INFINITY) continue;
      const float w = __expf(ls - m);
      tot += w;
      const float* src = p.Otail + (sl * 128 + r) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] += w * src[i];
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  const size_t o = ((size_t)tok * p.Hq + head) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(p.O) + o + i) =
        pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
  if (lane == 0) p.LSE[(size_t)head * p.L + tok] = tot > 0.f ? m + __logf(tot) : -INFINITY;
}

template <int D>
static cudaError_t launch_tile_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                 const AttnParams& p, int grid, cudaStream_t st) {
  using S = TileSmem<D>;
  static_assert(S::kAlloc <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(chunk_attn_tile_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
  if (e != cudaSuccess) return e;
  chunk_attn_tile_kernel<D><<<grid, kTThreads, S::kAlloc, st>>>(q, k, v, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.tail_k <= 1 || p.n_tail <= 0) return e;
  return launch_tail_combine(p, D, st);
}

cudaError_t launch_tail_combine(const AttnParams& p, int D, cudaStream_t st) {
  const dim3 grid(p.n_tail, 128 / 8);
  if (D == 128) tail_combine_kernel<128><<<grid, 256, 0, st>>>(p);
  else if (D == 64) tail_combine_kernel<64><<<grid, 256, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_chunk_attention_tile(const CUtensorMap& q, const CUtensorMap& k,
                                        const CUtensorMap& v, const AttnParams& p, int D,
                                        int grid, cudaStream_t st) {
  if (D == 128) return launch_tile_t<128>(q, k, v, p, grid, st);
  if (D == 64) return launch_tile_t<64>(q, k, v, p, grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace ca
