// internal.h — declarations shared by the library's translation units
// (kernel parameter block and host-side launchers).  Not part of the C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ca {

// One sequence's chunk inside a chunk-attention launch.  A single-sequence
// call carries one inline; a batch of sequences passes an array in device
// memory, ordered as the work units are (unit_start ascending).
struct SeqDesc {
  int q_start;     // first row of the chunk in Q / O, and column in LSE
  int L;           // chunk tokens
  int P;           // prefix tokens already in the cache (any value >= 0)
  int nKblk;       // ceil((P + L) / B): entries of its page table and table rows
  int pt_off;      // its page table starts at page_table[pt_off]; its tables at Hkv * pt_off
  int unit_start;  // its first work unit
  int nqs;         // ceil(L / 64) query spans
  int seq;         // its index in the caller's order (row of counts)
};

// Parameters of one chunk-attention launch (see chunk_attention.cu).
struct AttnParams {
  const int32_t* page_table;
  const int32_t* tables;
  const int32_t* counts;
  void* O;           // [L, Hq, D] bf16 or fp32 (n_splits == 1); L = all rows
  float* LSE;        // [Hq, L]                (n_splits == 1)
  float* Opart;      // [S, L, Hq, D] fp32      (n_splits > 1)
  float* LSEpart;    // [S, Hq, L] fp32         (n_splits > 1)
  int32_t* err;      // device error word (may be null)
  // persistent (stream-K) mode: each of sk_ctas CTAs takes an equal range of
  // all units' KV stages; split units leave fp32 partials for sk_combine
  int32_t* sk_sched;  // [n_units + 1] prefix of per-unit stage counts (written by CTA 0)
  float* Osk;         // [2 * sk_ctas][NT*128][D]
  float* LSEsk;       // [2 * sk_ctas][NT*128]
  int persistent, n_units, sk_ctas;
  const int32_t* n_units_dev;  // batched calls: the exact unit count (the grid is a bound)
  // fused mode (mask_bits != null): each CTA builds its group's table from the
  // bit-packed masks [Hq, nQblk_mask, mask_words] instead of reading tables;
  // one CTA per group writes it to tables_out / counts_out (either may be null)
  const uint32_t* mask_bits;
  int mask_words, nQblk_mask;
  int32_t* tables_out;
  int32_t* counts_out;
  // E4M3 pages: per table entry (group g, entry e) the (K, V) scales of its
  // page, escale[g * nKblk + e] (built by a gather kernel before the launch)
  const float2* escale;
  // tile kernel, split tail: units [tail_start, tail_start + n_tail) run as
  // tail_k pieces each (the last partial wave), leaving fp32 partials that a
  // merge kernel combines; all earlier units run whole
  int tail_start, tail_k, n_tail;
  float* Otail;    // [n_tail * tail_k][128][D]
  float* LSEtail;  // [n_tail * tail_k][128]
  const SeqDesc* seqs;  // [num_seqs] in device memory, or null: one sequence, seq0
  SeqDesc seq0;
  int num_seqs;
  int Hq, Hkv, G, HPU, nhalves, L, B, num_pages, n_splits, out_f32;  // L = rows of Q / O
  // order of the units within a sequence: 0 = by query span (later spans, with
  // more causal blocks, first), 1 = by KV group (all spans of a group together,
  // so the pages live in L2 at one time are those of few groups)
  int unit_order;
  float scale_log2;  // log2(e) / sqrt(D)
  unsigned long long wait_ns;
};

cudaError_t launch_build_tables(const uint8_t* mask, int nb, int Hq, int Hkv, int nQblk,
                                int nKblk, int32_t* tables, int32_t* counts, cudaStream_t stream);
cudaError_t launch_build_tables_bits(const uint32_t* bits, int nb, int Hq, int Hkv, int nQblk,
                                     int nKblk, int32_t* tables, int32_t* counts,
                                     cudaStream_t stream);
cudaError_t launch_chunk_attention(const CUtensorMap& q, const CUtensorMap& qlo,
                                   const CUtensorMap& k, const CUtensorMap& v,
                                   const AttnParams& p, int D, int NT, bool qsplit, bool kv8,
                                   int grid, cudaStream_t st);
// One 128-row tile per CTA, score tile triple-buffered in TMEM (bf16 only);
// launches the tail merge as well when p.tail_k > 1.
cudaError_t launch_chunk_attention_tile(const CUtensorMap& q, const CUtensorMap& k,
                                        const CUtensorMap& v, const AttnParams& p, int D,
                                        int grid, cudaStream_t st);
// CTA pairs (cta_group::2 MMAs of M = 256), head_dim 128, an even number of
// units (two head pairs per span); launches the tail merge as well.
cudaError_t launch_chunk_attention_pair(const CUtensorMap& q, const CUtensorMap& k,
                                        const CUtensorMap& v, const AttnParams& p, int D,
                                        int grid, cudaStream_t st);
// Merge the KV pieces of the split tail units (one-tile and pair kernels).
cudaError_t launch_tail_combine(const AttnParams& p, int D, cudaStream_t st);
cudaError_t launch_cast_bf16_f16(const void* src, void* dst, size_t n, cudaStream_t st);
cudaError_t launch_gather_scales(const int32_t* tables, const int32_t* counts,
                                 const int32_t* page_table, const float* K_scale,
                                 const float* V_scale, int Hkv, int nKblk, int num_pages,
                                 float2* escale, int32_t* err, cudaStream_t st);
cudaError_t launch_sk_combine(const AttnParams& p, int D, int NT, cudaStream_t st);
cudaError_t launch_split_combine(const float* Opart, const float* LSEpart, int n_splits, int L,
                                 int Hq, int D, void* O, float* LSE, int out_f32,
                                 cudaStream_t st);
cudaError_t launch_varlen_setup(const int32_t* cu_q, const int32_t* prefix_len,
                                const int32_t* cu_pages, int num_seqs, int total_q, int B, int Hkv,
                                int nhalves, SeqDesc* out, int32_t* n_units, int32_t* err,
                                cudaStream_t st);
cudaError_t launch_cast_f32_bf16(const float* src, void* dst, size_t n, cudaStream_t st);
cudaError_t launch_split_f32_bf16(const float* src, void* hi, void* lo, size_t n,
                                  cudaStream_t st);
cudaError_t launch_wait_probe(int32_t* err, unsigned long long limit_ns, cudaStream_t st);

// Streaming multiprocessors of the calling thread's current device (148 when
// no device can be queried).
int num_sms();

// Record a message for ca_last_error() on the calling thread.
void set_last_error(const char* msg);

}  // namespace ca
