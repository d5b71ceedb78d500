// internal.h — declarations shared by the library's translation units
// (kernel parameter block and host-side launchers).  Not part of the C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ca {

// Parameters of one chunk-attention launch (see chunk_attention.cu).
struct AttnParams {
  const int32_t* page_table;
  const int32_t* tables;
  const int32_t* counts;
  void* O;           // [L, Hq, D] bf16 or fp32 (n_splits == 1)
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
  int Hq, Hkv, G, HPU, nhalves, L, P, B, nPblk, nKblk, num_pages, n_splits, nqs, out_f32;
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
                                   const AttnParams& p, int D, int NT, bool qsplit, int grid,
                                   cudaStream_t st);
cudaError_t launch_sk_combine(const AttnParams& p, int D, int NT, cudaStream_t st);
cudaError_t launch_split_combine(const float* Opart, const float* LSEpart, int n_splits, int L,
                                 int Hq, int D, void* O, float* LSE, int out_f32,
                                 cudaStream_t st);
cudaError_t launch_cast_f32_bf16(const float* src, void* dst, size_t n, cudaStream_t st);
cudaError_t launch_split_f32_bf16(const float* src, void* hi, void* lo, size_t n,
                                  cudaStream_t st);
cudaError_t launch_wait_probe(int32_t* err, unsigned long long limit_ns, cudaStream_t st);

// Record a message for ca_last_error() on the calling thread.
void set_last_error(const char* msg);

}  // namespace ca
