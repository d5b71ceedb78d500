// append_kv.cu — write a prefill chunk's new keys and values into the paged
// KV cache, in place, through the page table.
//
// "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
// Selection", Abstract: chunked prefill grows the accumulated KV cache chunk
// by chunk and the cache is read in place under paged execution; this is the
// write side of that cache.  Token i of the chunk sits at position
// p = prefix_len + i, in logical block p / B, physical page page_table[p / B],
// row p % B.  The rows of the last block after the chunk's last position are
// zero-filled, so that the attention kernel, which multiplies every row of a
// fetched block (by a zero weight past the sequence end), never meets stale
// non-finite data.  Bandwidth-bound: each 16-byte vector is read once and
// written once; a thread moves one vector of K and the same vector of V.
#include <cuda_runtime.h>

#include <cstdint>

#include "compactattn.h"
#include "internal.h"

namespace ca {

__global__ void __launch_bounds__(256)
    append_kv_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                     uint4* __restrict__ k_pages, uint4* __restrict__ v_pages,
                     const int32_t* __restrict__ page_table, int prefix_len, int chunk_len,
                     int Hkv, int vec_per_row, int block, int num_pages, int nKblk, int tail,
                     int32_t* err) {
  // 32-bit index math (the host bounds the vector count below 2^31)
  const unsigned total = (unsigned)(chunk_len + tail) * (unsigned)Hkv * (unsigned)vec_per_row;
  for (unsigned idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += gridDim.x * blockDim.x) {
    const unsigned v = idx % (unsigned)vec_per_row;
    const unsigned rg = idx / (unsigned)vec_per_row;
    const int g = (int)(rg % (unsigned)Hkv);
    const int i = (int)(rg / (unsigned)Hkv);
    const int pos = prefix_len + i;
    const int kb = pos / block;
    int page = (kb < nKblk) ? page_table[kb] : -1;
    if (page < 0 || page >= num_pages) {
      if (err) atomicOr(err, CA_FLAG_BOUNDS);
      continue;  // never write outside the cache
    }
    const size_t dst = (((size_t)page * Hkv + g) * block + pos % block) * vec_per_row + v;
    if (i < chunk_len) {
      k_pages[dst] = __ldcs(k_new + idx);
      v_pages[dst] = __ldcs(v_new + idx);
    } else {
      k_pages[dst] = make_uint4(0u, 0u, 0u, 0u);
      v_pages[dst] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

cudaError_t launch_append_kv(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                             const int32_t* page_table, int prefix_len, int chunk_len, int Hkv,
                             int row_bytes, int block, int num_pages, int nKblk, int32_t* err,
                             cudaStream_t st) {
  const int vec = row_bytes / 16;
  const int end = prefix_len + chunk_len;
  const int tail = chunk_len > 0 ? (block - end % block) % block : 0;  // rest of the last block
  const long long total = (long long)(chunk_len + tail) * Hkv * vec;
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  append_kv_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      static_cast<uint4*>(k_pages), static_cast<uint4*>(v_pages), page_table, prefix_len,
      chunk_len, Hkv, vec, block, num_pages, nKblk, tail, err);
  return cudaGetLastError();
}

}  // namespace ca

extern "C" int ca_append_kv(const void* K_new, const void* V_new, int dtype, void* K_pages,
                            void* V_pages, int num_pages, const int32_t* page_table, int Hkv,
                            int head_dim, int block, int prefix_len, int chunk_len,
                            int32_t* err_flag, void* stream) {
  // An empty chunk writes nothing; its row buffers may then be NULL.
  if ((chunk_len > 0 && (!K_new || !V_new)) || !K_pages || !V_pages || !page_table) {
    ca::set_last_error("ca_append_kv: null pointer");
    return CA_ERR_ARG;
  }
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32) {
    ca::set_last_error("ca_append_kv: dtype code not supported");
    return CA_ERR_DTYPE;
  }
  const int esize = dtype == CA_DTYPE_BF16 ? 2 : 4;
  if (Hkv < 1 || head_dim < 1 || block < 1 || prefix_len < 0 || chunk_len < 0 ||
      (head_dim * esize) % 16) {
    ca::set_last_error("ca_append_kv: bad shape (head_dim * element size must be a multiple of 16)");
    return CA_ERR_ARG;
  }
  const long long nKblk = ((long long)prefix_len + chunk_len + block - 1) / block;
  if (nKblk > num_pages || nKblk > 0x7fffffffLL) {
    ca::set_last_error("ca_append_kv: the chunk's blocks exceed num_pages");
    return CA_ERR_ARG;
  }
  if ((long long)(chunk_len + block) * Hkv * (head_dim * esize / 16) >= 0x7fffffffLL) {
    ca::set_last_error("ca_append_kv: chunk too large for one call");
    return CA_ERR_ARG;
  }
  const uintptr_t al = reinterpret_cast<uintptr_t>(K_new) | reinterpret_cast<uintptr_t>(V_new) |
                       reinterpret_cast<uintptr_t>(K_pages) | reinterpret_cast<uintptr_t>(V_pages);
  if (al & 15u) {
    ca::set_last_error("ca_append_kv: buffers must be 16-byte aligned");
    return CA_ERR_ARG;
  }
  cudaError_t e = ca::launch_append_kv(K_new, V_new, K_pages, V_pages, page_table, prefix_len,
                                       chunk_len, Hkv, head_dim * esize, block, num_pages,
                                       (int)nKblk, err_flag, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    ca::set_last_error("ca_append_kv: launch failed");
    return CA_ERR_LAUNCH;
  }
  return CA_OK;
}
