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
// fetched from HBM/L2 feeds 2*NT MMAs.  Because the chunk starts on a block
// boundary, the blocks a span may see are a prefix of the sorted table
// (entries <= the span's diagonal block), and only the diagonal block needs a
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
#include <cuda_runtime.h>

#include <cstdint>

#include "compactattn.h"
#include "internal.h"
#include "ptx.cuh"

namespace ca {

constexpr int kStageKeys = 128;



__device__ __forceinline__ void set_flag(int32_t* err, int f) {
  if (err) atomicOr(err, f);
}

// QSPLIT: Q is given as two bf16 terms (hi + lo) of an fp32 input and
// S = Q_hi K^T + Q_lo K^T, which removes the rounding error of Q (the error
// term shared by all keys of a row); used for fp32 inputs.
template <int D, int NT, bool QSPLIT>
struct Smem {
  static constexpr int kQTerms = QSPLIT ? 2 : 1;
  static constexpr int kChunkBytes = 128 * 128;         // 128 rows x 128 B (64 bf16)
  static constexpr int kQTile = 128 * D * 2;            // one 128-row Q tile
  static constexpr int kKV = kStageKeys * D * 2;        // one stage of K (or V)
  // K/V ring depth: two stages unless the split Q tiles leave room for one only
  static constexpr int kNS = (kQTerms * NT * kQTile + 4 * kKV <= 200 * 1024) ? 2 : 1;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQTerms * NT * kQTile;
  static constexpr int kVOff = kKOff + kNS * kKV;
  static constexpr int kBarOff = kVOff + kNS * kKV;
  // barriers: q_full, full_k[NS], full_v[NS], empty_k[NS], empty_v[NS],
  //           s_full[2], p_full[2], o_done, drain
  static constexpr int kNumBars = 1 + 4 * kNS + 2 + 2 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 64;
  static constexpr int kAlloc = kBytes + 1024;          // slack for 1024-B alignment
};

// Warp-uniform bounded wait.  Returns false (and flags / aborts) on expiry.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const AttnParams& p,
                                          volatile int* abort_flag) {
  bool ok = (*abort_flag == 0) && mbar_wait(bar, parity, p.wait_ns);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) {
    if ((threadIdx.x & 31) == 0 && *abort_flag == 0) {
      *abort_flag = 1;
      set_flag(p.err, CA_FLAG_TIMEOUT);
    }
  }
  return ok;
}

template <int D, int NT, bool QSPLIT>
__global__ void __launch_bounds__(128 + NT * 128, 1)
    chunk_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmQlo,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using S = Smem<D, NT, QSPLIT>;
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
  int* misc = reinterpret_cast<int*>(sm + S::kMiscOff);
  // misc[0] tmem base, [1] n_live, [2] has_diag, [3] first stage, [4] stage count, [5] abort
  volatile int* abort_flag = misc + 5;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- decode the work item (heaviest query spans first)
  const int item = blockIdx.x;
  const int split = item % p.n_splits;
  const int unit = item / p.n_splits;
  const int per_qs = p.Hkv * p.nhalves;
  const int qs = p.nqs - 1 - unit / per_qs;
  const int g = (unit % per_qs) / p.nhalves;
  const int hh = (unit % per_qs) % p.nhalves;
  const int t0 = qs * 64;
  const int diag_kb = p.nPblk + t0 / p.B;
  const int spb = kStageKeys / p.B;  // pages per stage
  const int32_t* trow = p.tables + (size_t)g * p.nKblk;

  if (threadIdx.x == 0) {
    int cnt = p.counts[g];
    if (cnt < 0 || cnt > p.nKblk) {
      set_flag(p.err, CA_FLAG_BOUNDS);
      cnt = cnt < 0 ? 0 : p.nKblk;
    }
    int lo = 0, hi = cnt;  // entries <= diag_kb form a prefix of the sorted row
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (trow[mid] <= diag_kb) lo = mid + 1;
      else hi = mid;
    }
    const int n_live = lo;
    const int nst = (n_live + spb - 1) / spb;
    const int s0 = (int)((long long)split * nst / p.n_splits);
    const int s1 = (int)((long long)(split + 1) * nst / p.n_splits);
    misc[1] = n_live;
    misc[2] = (n_live > 0 && trow[n_live - 1] == diag_kb) ? 1 : 0;
    misc[3] = s0;
    misc[4] = s1 - s0;
    misc[5] = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(full_k(s), 1);
      mbar_init(full_v(s), 1);
      mbar_init(empty_k(s), 1);
      mbar_init(empty_v(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 4);  // one arrival per softmax warp
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
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
  const int n_live = misc[1];
  const int has_diag = misc[2];
  const int s0 = misc[3];
  const int nloc = misc[4];
  const int nst_total = (n_live + spb - 1) / spb;

  if (warp == 0) {
    // ================================================================ producer
    // The whole warp runs the loop: lane i prefetches table entry i of the next
    // group of 32 and its page id, so the dependent lookups tables ->
    // page_table are off the per-stage path; lane 0 issues the copies.
    if (nloc > 0) {
      const uint64_t pol = policy_evict_last();
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        if (QSPLIT) prefetch_tmap(&tmQlo);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        mbar_expect_tx(q_full, S::kQTerms * NT * 128 * D * 2);
        for (int q = 0; q < S::kQTerms; ++q)
          for (int t = 0; t < NT; ++t)
            for (int s = 0; s < 2; ++s) {
              int hl = hh * p.HPU + 2 * t + s;  // head within the group
              const int hcap = min(p.G - 1, hh * p.HPU + p.HPU - 1);
              hl = min(hl, hcap);
              const int head = g * p.G + hl;
              for (int c = 0; c < KCH; ++c)
                tma_load_3d(sbase + S::kQOff + (q * NT + t) * S::kQTile + c * S::kChunkBytes +
                                s * 64 * 128,
                            q ? &tmQlo : &tmQ, q_full, c * 64, head, t0);
            }
      }
      const int e_begin = s0 * spb;
      const int e_end = min(n_live, (s0 + nloc) * spb);
      int pg_cache = 0, cache_base = -32;
      bool ok = true;
      for (int j = 0; j < nloc && ok; ++j) {
        const int stage = s0 + j, slot = j % kNS, round = j / kNS;
        const int npg = min(spb, n_live - stage * spb);
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
              if (kb < 0 || kb >= p.nKblk) {
                set_flag(p.err, CA_FLAG_BOUNDS);
                kb = 0;
              }
              pg = p.page_table[kb];
              if (pg < 0 || pg >= p.num_pages) {
                set_flag(p.err, CA_FLAG_BOUNDS);
                pg = 0;
              }
            }
            pg_cache = pg;
          }
          page[pi] = __shfl_sync(0xffffffffu, pg_cache, e - cache_base);
        }
        if (round > 0) ok = wait_warp(empty_k(slot), (round - 1) & 1, p, abort_flag);
        if (ok) {
          mbar_expect_tx_w(full_k(slot), bytes);
          for (int pi = 0; pi < npg; ++pi)
            for (int c = 0; c < KCH; ++c)
              tma_load_4d_w(sbase + S::kKOff + slot * S::kKV + c * S::kChunkBytes + pi * p.B * 128,
                            &tmK, full_k(slot), c * 64, 0, g, page[pi], pol);
        }
        if (ok && round > 0) ok = wait_warp(empty_v(slot), (round - 1) & 1, p, abort_flag);
        if (ok) {
          mbar_expect_tx_w(full_v(slot), bytes);
          for (int pi = 0; pi < npg; ++pi)
            for (int c = 0; c < KCH; ++c)
              tma_load_4d_w(sbase + S::kVOff + slot * S::kKV + c * S::kChunkBytes + pi * p.B * 128,
                            &tmV, full_v(slot), c * 64, 0, g, page[pi], pol);
        }
      }
      if (lane == 0) {
        // Do not leave with copies in flight: the last stages' loads must land.
        for (int j = max(0, nloc - kNS); j < nloc; ++j) {
          mbar_wait(full_k(j % kNS), (j / kNS) & 1, p.wait_ns);
          mbar_wait(full_v(j % kNS), (j / kNS) & 1, p.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // The whole warp runs this loop (addresses stay warp-uniform); one elected
    // lane issues each tcgen05.mma / commit.
    if (nloc > 0) {
      // Descriptors differ per MMA only in the start-address field (address >> 4
      // in bits 0-13): build each operand's descriptor once and add the
      // compile-time byte offset >> 4 per K-step.
      constexpr uint32_t kIdescPV = idesc_bf16(128, D, 1);
      constexpr uint32_t kIdescS128 = idesc_bf16(128, 128, 0);
      constexpr uint32_t kIdescS64 = idesc_bf16(128, 64, 0);
      uint64_t qdesc[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) qdesc[t] = smem_desc_sw128(sbase + S::kQOff + t * S::kQTile, 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(sbase + S::kKOff, 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(sbase + S::kVOff, S::kChunkBytes, 1024);
      auto npg_of = [&](int j) { return min(spb, n_live - (s0 + j) * spb); };
      auto issue_s = [&](int t, int j) {
        const uint64_t kd = kdesc0 + (uint64_t)(((j % kNS) * S::kKV) >> 4);
        const uint32_t idesc = npg_of(j) * p.B == 128 ? kIdescS128 : kIdescS64;
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
        const uint64_t vd = vdesc0 + (uint64_t)(((j % kNS) * S::kKV) >> 4);
        const uint32_t dt = tmem + t * 128;
        const uint32_t at = tmem + 256 + t * 128;
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        if (npg_of(j) * p.B == 128) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(dt, at + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV, kk > 0 ? 1u : acc0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts_w(dt, at + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescPV, kk > 0 ? 1u : acc0);
        }
      };
      bool ok = wait_warp(q_full, 0, p, abort_flag) && wait_warp(full_k(0), 0, p, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit_w(s_full(0));
        if (NT == 2) {
          issue_s(1, 0);
          mma_commit_w(s_full(1));
        }
        mma_commit_w(empty_k(0));
      }
      for (int j = 0; j < nloc && ok; ++j) {
        const int slot = j % kNS;
        ok = wait_warp(p_full(0), j & 1, p, abort_flag) &&
             wait_warp(full_v(slot), (j / kNS) & 1, p, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, j);
        const bool more = j + 1 < nloc;
        if (more) {
          ok = wait_warp(full_k((j + 1) % kNS), ((j + 1) / kNS) & 1, p, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, j + 1);
          mma_commit_w(s_full(0));
        }
        if (NT == 2) {
          ok = wait_warp(p_full(1), j & 1, p, abort_flag);
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
          mma_commit_w(empty_k((j + 1) % kNS));
        }
      }
      if (ok) mma_commit_w(o_done);
      // every MMA issued by this warp has finished before TMEM is released
      mma_commit_w(drain);
      mbar_wait(drain, 0, p.wait_ns);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax / epilogue
    const int t = (warp - 4) >> 2;
    const int row = threadIdx.x & 127;
    const int sub = row >> 6;
    const int tok = t0 + (row & 63);
    const int hl_raw = hh * p.HPU + 2 * t + sub;
    const bool valid_row = (2 * t + sub) < p.HPU && hl_raw < p.G;
    const int head = g * p.G + min(hl_raw, p.G - 1);
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + 256 + t * 128;
    const uint32_t tO = tmem + lane_off + t * 128;
    const int diag_lim = (t0 % p.B) + (row & 63);  // visible keys of the diagonal block: jl <= this
    float m_used = -INFINITY, l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
    bool ok = true;
    for (int j = 0; j < nloc; ++j) {
      const int stage = s0 + j;
      const int npg = min(spb, n_live - stage * spb);
      const int nvalid = npg * p.B;
      const bool diag_stage = has_diag && (stage == nst_total - 1);
      const int diag_c0 = (npg - 1) * p.B;  // first column of the diagonal page
      ok = wait_warp(s_full(t), j & 1, p, abort_flag);
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
      if (diag_stage) {  // token-level causal mask, diagonal block only
#pragma unroll
        for (int c = 0; c < kStageKeys; ++c)
          if (c >= diag_c0 && (c - diag_c0) > diag_lim) sr[c] = -INFINITY;
      }
      // row max of the raw scores (scale > 0 commutes with max)
      float mx0 = max3(sr[0], sr[1], sr[2]);
      float mx1 = max3(sr[3], sr[4], sr[5]);
#pragma unroll
      for (int c = 6; c < kStageKeys - 2; c += 4) {
        mx0 = max3(mx0, sr[c], sr[c + 1]);
        mx1 = max3(mx1, sr[c + 2], sr[c + 3]);
      }
      const float mx = max3(mx0, mx1, fmaxf(sr[kStageKeys - 2], sr[kStageKeys - 1])) * p.scale_log2;
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
    // ---- epilogue
    const float l = (l0 + l1) + (l2 + l3);
    if (ok && nloc > 0) ok = wait_warp(o_done, 0, p, abort_flag);
    if (ok && nloc > 0) tc_fence_after();
    const bool have = ok && nloc > 0 && l > 0.f;
    const float inv = have ? 1.f / l : 0.f;
    const float lse = have ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    const bool split_out = p.n_splits > 1;
    uint32_t r[32];
    for (int c = 0; c < D / 32; ++c) {
      if (ok && nloc > 0) {
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
      if (split_out) {
        float4* dst = reinterpret_cast<float4*>(
            p.Opart + (((size_t)split * p.L + tok) * p.Hq + head) * D + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      } else if (p.out_f32) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.O) +
                                                ((size_t)tok * p.Hq + head) * D + c * 32);
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
      if (split_out) p.LSEpart[((size_t)split * p.Hq + head) * p.L + tok] = lse;
      else p.LSE[(size_t)head * p.L + tok] = lse;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
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

template <int D, int NT, bool QS>
static cudaError_t launch_attn_t(const CUtensorMap& q, const CUtensorMap& qlo,
                                 const CUtensorMap& k, const CUtensorMap& v, const AttnParams& p,
                                 int grid, cudaStream_t st) {
  using S = Smem<D, NT, QS>;
  static_assert(S::kAlloc <= 227 * 1024, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(chunk_attn_kernel<D, NT, QS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
  if (e != cudaSuccess) return e;
  chunk_attn_kernel<D, NT, QS><<<grid, 128 + NT * 128, S::kAlloc, st>>>(q, qlo, k, v, p);
  return cudaGetLastError();
}

cudaError_t launch_chunk_attention(const CUtensorMap& q, const CUtensorMap& qlo,
                                   const CUtensorMap& k, const CUtensorMap& v,
                                   const AttnParams& p, int D, int NT, bool qsplit, int grid,
                                   cudaStream_t st) {
#define CA_LAUNCH(d_, nt_, qs_)                                                  \
  if (D == d_ && NT == nt_ && qsplit == qs_)                                     \
    return launch_attn_t<d_, nt_, qs_>(q, qlo, k, v, p, grid, st);
  CA_LAUNCH(128, 2, false)
  CA_LAUNCH(128, 1, false)
  CA_LAUNCH(64, 2, false)
  CA_LAUNCH(64, 1, false)
  CA_LAUNCH(128, 2, true)
  CA_LAUNCH(128, 1, true)
  CA_LAUNCH(64, 2, true)
  CA_LAUNCH(64, 1, true)
#undef CA_LAUNCH
  return cudaErrorInvalidValue;
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
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  cast_f32_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, reinterpret_cast<__nv_bfloat16*>(dst), n);
  return cudaGetLastError();
}

cudaError_t launch_split_f32_bf16(const float* src, void* hi, void* lo, size_t n,
                                  cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  split_f32_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      src, reinterpret_cast<__nv_bfloat16*>(hi), reinterpret_cast<__nv_bfloat16*>(lo), n);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(int32_t* err, unsigned long long limit_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace ca
