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

// Block (row i, head-group y): threadIdx.x = 16-byte vector of a head's row,
// threadIdx.y = head within the block's group of heads; no index division.
__global__ void __launch_bounds__(256)
    append_kv_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                     uint4* __restrict__ k_pages, uint4* __restrict__ v_pages,
                     const int32_t* __restrict__ page_table, int prefix_len, int chunk_len,
                     int Hkv, int vec_per_row, int block, int num_pages, int nKblk,
                     int32_t* err) {
  const int i = blockIdx.x;  // token of the chunk, or of the cleared tail past it
  const int g = blockIdx.y * blockDim.y + threadIdx.y;
  const int v = threadIdx.x;
  if (g >= Hkv) return;
  const int pos = prefix_len + i;
  const int kb = pos / block;
  const int page = (kb < nKblk) ? page_table[kb] : -1;
  if (page < 0 || page >= num_pages) {
    if (err && v == 0) atomicOr(err, CA_FLAG_BOUNDS);
    return;  // never write outside the cache
  }
  const size_t dst = (((size_t)page * Hkv + g) * block + pos % block) * vec_per_row + v;
  if (i < chunk_len) {
    const size_t src = ((size_t)i * Hkv + g) * vec_per_row + v;
    k_pages[dst] = __ldcs(k_new + src);
    v_pages[dst] = __ldcs(v_new + src);
  } else {
    k_pages[dst] = make_uint4(0u, 0u, 0u, 0u);
    v_pages[dst] = make_uint4(0u, 0u, 0u, 0u);
  }
}

cudaError_t launch_append_kv(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                             const int32_t* page_table, int prefix_len, int chunk_len, int Hkv,
                             int row_bytes, int block, int num_pages, int nKblk, int32_t* err,
                             cudaStream_t st) {
  const int vec = row_bytes / 16;
  const int end = prefix_len + chunk_len;
  const int tail = chunk_len > 0 ? (block - end % block) % block : 0;  // rest of the last block
  const int rows = chunk_len + tail;
  if (rows == 0) return cudaSuccess;
  int hy = 256 / vec;  // heads per block
  if (hy < 1) hy = 1;
  if (hy > Hkv) hy = Hkv;
  const dim3 blk(vec, hy), grid(rows, (Hkv + hy - 1) / hy);
  append_kv_kernel<<<grid, blk, 0, st>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      static_cast<uint4*>(k_pages), static_cast<uint4*>(v_pages), page_table, prefix_len,
      chunk_len, Hkv, vec, block, num_pages, nKblk, err);
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
  if (head_dim * esize / 16 > 256 || (long long)chunk_len + block > 0x7fffffffLL) {
    ca::set_last_error("ca_append_kv: row or chunk too large for one call");
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
