// capi.cu — the extern "C" boundary of libcompactattn.so: argument checks,
// TMA tensor maps over the paged KV cache, work/split planning, launches and
// error reporting.  The call signatures are declared and documented in
// include/compactattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "compactattn.h"
#include "internal.h"

namespace ca {
namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(CA_ERR_LAUNCH, "%s: %s", what, cudaGetErrorString(e));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per pipeline wait

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kMaxPersistentUnits = 2048;  // units whose schedule a CTA keeps in shared memory

struct Plan {
  int G, HPU, NT, nhalves, spb, n_splits;
  int units, persistent, sk_ctas;
  int tile;                          // 1: the one-tile kernel (bf16 pages and Q)
  int pair;                          // 1: the CTA-pair kernel (bf16, head_dim 128, even units)
  int tail_start, tail_k, n_tail;    // tile kernel: the split last partial wave
};

// Heads -> tiles.  Two-tile kernel: a unit stacks up to four heads of a group
// over a 64-token span (two heads per 128-row tile).  One-tile kernel: a unit
// is two heads of a group over a 64-token span, one 128-row tile.
bool plan_heads(int Hq, int Hkv, int head_dim, int block, Plan& pl, bool tile = false) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return false;
  if (head_dim != 64 && head_dim != 128) return false;
  if (block != 64 && block != 128) return false;
  pl.G = Hq / Hkv;
  pl.tile = tile ? 1 : 0;
  if (tile) {
    pl.HPU = pl.G < 2 ? pl.G : 2;
    pl.NT = 1;
    pl.nhalves = (pl.G + 1) / 2;
  } else {
    pl.HPU = pl.G < 4 ? pl.G : 4;
    pl.NT = (pl.HPU + 1) / 2;
    pl.nhalves = (pl.G + pl.HPU - 1) / pl.HPU;
  }
  pl.spb = 128 / block;
  // CTA pairs take the two head pairs of a group's span together: head_dim
  // 128 and an even number of head pairs per group (G = 3, 4, 7, 8, ...)
  pl.pair = (tile && head_dim == 128 && pl.nhalves % 2 == 0) ? 1 : 0;
  pl.tail_start = 0;
  pl.tail_k = 1;
  pl.n_tail = 0;
  return true;
}

// Work mode of the one-tile kernel for `units` units of at most `max_stages`
// KV stages each (one CTA per SM).  n_splits > 0: every unit in that many KV
// pieces.  Automatic (n_splits <= 0): with fewer units than SMs, every unit in
// floor(SMs / units) pieces (at most 16), so that one wave fills the SMs;
// otherwise one CTA per unit, and when the units are known exactly the r
// units of the last partial wave run as k pieces each, k the largest with
// r * k <= SMs (at most 4): the last wave then takes 1/k of a unit's time.
bool plan_mode_tile(Plan& pl, long long units, int max_stages, int n_splits, bool exact_units) {
  if (units > 0x7fffffffLL) return false;
  pl.units = (int)units;
  pl.persistent = 0;
  pl.sk_ctas = 0;
  pl.tail_start = (int)units;
  pl.tail_k = 1;
  pl.n_tail = 0;
  // the pair kernel places a pair of units on a pair of SMs
  const long long per = pl.pair ? 2 : 1;
  const long long sms = num_sms() / per, jobs = units / per;
  long long S = n_splits;
  if (S <= 0) {
    S = jobs > 0 && jobs < sms ? std::min<long long>(16, std::max<long long>(1, sms / jobs)) : 1;
    const long long r = jobs % sms;
    if (exact_units && jobs >= sms && r > 0) {
      const int k = (int)std::min<long long>({4, sms / r, (long long)max_stages});
      if (k >= 2) {
        pl.tail_k = k;
        pl.n_tail = (int)(r * per);
        pl.tail_start = (int)(units - r * per);
      }
    }
  }
  if (S > max_stages) S = max_stages;
  if (S < 1) S = 1;
  if (units * S > 0x7fffffffLL) return false;
  pl.n_splits = (int)S;
  return true;
}

// Grid of an attention launch for plan pl.
int plan_grid(const Plan& pl) {
  if (pl.persistent) return pl.sk_ctas;
  if (pl.tile && pl.tail_k > 1) return pl.tail_start + pl.n_tail * pl.tail_k;
  return pl.units * pl.n_splits;
}

// Work mode for `units` units of at most `max_stages` KV stages each.
bool plan_mode(Plan& pl, long long units, int max_stages, int n_splits, bool allow_persistent) {
  if (units > 0x7fffffffLL) return false;
  pl.units = (int)units;
  // Automatic mode: one CTA per unit when the units fill the SMs; otherwise a
  // persistent grid of at most one CTA per SM, each taking an equal share of
  // all units' KV stages (at least ~4 stages per CTA).  (At 256 units on 148
  // SMs the persistent grid measured 5% slower than one CTA per unit: the
  // piece boundaries and the merge cost more than the balance gains.)
  const int sms = num_sms();
  pl.persistent = (allow_persistent && n_splits <= 0 && units < sms && units <= kMaxPersistentUnits)
                      ? 1 : 0;
  if (n_splits <= 0 && !pl.persistent) n_splits = 1;
  pl.sk_ctas = 0;
  if (pl.persistent) {
    const long long stages = units * max_stages;
    pl.sk_ctas = (int)std::max<long long>(1, std::min<long long>(sms, stages / 4));
    pl.n_splits = 1;
    return true;
  }
  int S = n_splits;
  if (S > max_stages) S = max_stages;
  if (S < 1) S = 1;
  if (units * S > 0x7fffffffLL) return false;
  pl.n_splits = S;
  return true;
}

// One sequence: chunk_len >= 1 tokens after prefix_len >= 0 tokens (no
// alignment needed: masks hold Q-blocks of the chunk's tokens and KV blocks
// of the sequence's positions).
bool plan(int Hq, int Hkv, int head_dim, int block, int chunk_len, int prefix_len, int n_splits,
          Plan& pl, SeqDesc& d, bool tile = false) {
  if (!plan_heads(Hq, Hkv, head_dim, block, pl, tile)) return false;
  if (chunk_len < 1 || prefix_len < 0 || (long long)prefix_len + chunk_len > 0x7fffffffLL)
    return false;
  d.q_start = 0;
  d.L = chunk_len;
  d.P = prefix_len;
  d.nKblk = (int)(((long long)prefix_len + chunk_len + block - 1) / block);
  d.pt_off = 0;
  d.unit_start = 0;
  d.nqs = (chunk_len + 63) / 64;
  d.seq = 0;
  const long long units = (long long)Hkv * pl.nhalves * d.nqs;
  const int max_stages = (d.nKblk + pl.spb - 1) / pl.spb;
  if (tile) return plan_mode_tile(pl, units, max_stages, n_splits, true);
  return plan_mode(pl, units, max_stages, n_splits, true);
}

struct WsLayout {
  size_t opart = 0, lsepart = 0, q = 0, qlo = 0, k = 0, v = 0, sched = 0, osk = 0, lsesk = 0,
         seqs = 0, nunits = 0, q16 = 0, esc = 0, otail = 0, lsetail = 0, total = 0;
};

// rows = rows of Q / O; num_seqs > 0 reserves the batched call's descriptors.
WsLayout ws_layout(int dtype, int Hq, int Hkv, int D, int B, long long rows, int num_pages,
                   const Plan& pl, int num_seqs = 0, int nKblk_e4m3 = 0) {
  WsLayout w;
  size_t off = 0;
  const int S = pl.n_splits;
  if (num_seqs > 0) {
    w.seqs = off;
    off = align256(off + (size_t)num_seqs * sizeof(SeqDesc));
    w.nunits = off;
    off = align256(off + 4);
  }
  if (pl.persistent) {
    const size_t trows = (size_t)pl.NT * 128;
    w.sched = off;
    off = align256(off + (size_t)(pl.units + 1) * 4);
    w.osk = off;
    off = align256(off + 2 * (size_t)pl.sk_ctas * trows * D * 4);
    w.lsesk = off;
    off = align256(off + 2 * (size_t)pl.sk_ctas * trows * 4);
  }
  if (pl.tile && pl.tail_k > 1) {
    const size_t pieces = (size_t)pl.n_tail * pl.tail_k;
    w.otail = off;
    off = align256(off + pieces * 128 * D * 4);
    w.lsetail = off;
    off = align256(off + pieces * 128 * 4);
  }
  if (S > 1) {
    w.opart = off;
    off = align256(off + (size_t)S * rows * Hq * D * 4);
    w.lsepart = off;
    off = align256(off + (size_t)S * Hq * rows * 4);
  }
  if (dtype == CA_DTYPE_E4M3) {  // f16 copy of Q, per-entry page scales
    w.q16 = off;
    off = align256(off + (size_t)rows * Hq * D * 2);
    w.esc = off;
    off = align256(off + (size_t)Hkv * nKblk_e4m3 * 8);
  }
  if (dtype == CA_DTYPE_FP32) {
    w.q = off;
    off = align256(off + (size_t)rows * Hq * D * 2);
    w.qlo = off;
    off = align256(off + (size_t)rows * Hq * D * 2);
    w.k = off;
    off = align256(off + (size_t)num_pages * Hkv * B * D * 2);
    w.v = off;
    off = align256(off + (size_t)num_pages * Hkv * B * D * 2);
  }
  w.total = off;
  return w;
}

// Units bound of a batched call: sum_s ceil(L_s / 64) <= total_q / 64 + num_seqs.
long long varlen_units_bound(int total_q, int num_seqs, int Hkv, int nhalves) {
  return ((long long)(total_q + 63) / 64 + num_seqs) * Hkv * nhalves;
}

// Plan of a batched call (the exact unit count is only known on the device:
// the plan is made for the bound, and surplus CTAs leave at once).
bool plan_varlen(int Hq, int Hkv, int head_dim, int block, int dtype, int num_seqs, int total_q,
                 int max_kv_len, int n_splits, Plan& pl) {
  const bool tile = dtype == CA_DTYPE_BF16;
  if (!plan_heads(Hq, Hkv, head_dim, block, pl, tile)) return false;
  const int max_stages = std::max(1, (max_kv_len + 127) / 128);
  const long long bound = varlen_units_bound(total_q, num_seqs, Hkv, pl.nhalves);
  if (tile) return plan_mode_tile(pl, bound, max_stages, n_splits, false);
  return plan_mode(pl, bound, max_stages, n_splits, false);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

// Streaming multiprocessors of the calling thread's current device: the
// persistent grid and the automatic split plan are sized from it.  Without a
// usable device (a host-only size query) the B200's 148 is assumed; a plan made
// that way is checked again by the launching call, which needs the workspace
// its own device's plan asks for.
int num_sms() {
  static std::atomic<int> cache[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    (void)cudaGetLastError();
    return 148;
  }
  if (dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return 148;
  }
  if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}


}  // namespace ca

using namespace ca;

extern "C" {

int ca_version(void) { return 100; }

int ca_last_error(char* buf, size_t n) {
  if (!buf || n == 0) return CA_ERR_ARG;
  const size_t m = g_last_error.size() < n - 1 ? g_last_error.size() : n - 1;
  memcpy(buf, g_last_error.data(), m);
  buf[m] = 0;
  return CA_OK;
}

int ca_build_tables_batched(const uint8_t* masks, int nb, int Hq, int Hkv, int nQblk, int nKblk,
                            int32_t* tables, int32_t* counts, void* stream) {
  if (!masks || !tables || !counts) return fail(CA_ERR_ARG, "ca_build_tables: null pointer");
  if (nb < 1 || nb > 65535) return fail(CA_ERR_ARG, "ca_build_tables: nb=%d out of [1,65535]", nb);
  if (Hq < 1 || Hkv < 1 || Hkv > Hq || Hq % Hkv)
    return fail(CA_ERR_ARG, "ca_build_tables: Hq=%d must be a positive multiple of Hkv=%d", Hq, Hkv);
  if (Hkv > 65535) return fail(CA_ERR_ARG, "ca_build_tables: Hkv=%d too large", Hkv);
  if (nQblk < 1) return fail(CA_ERR_ARG, "ca_build_tables: nQblk=%d < 1", nQblk);
  if (nKblk < 1 || nKblk > 65536)
    return fail(CA_ERR_ARG, "ca_build_tables: nKblk=%d out of [1,65536]", nKblk);
  cudaError_t e = launch_build_tables(masks, nb, Hq, Hkv, nQblk, nKblk, tables, counts,
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "ca_build_tables launch");
  return CA_OK;
}

int ca_build_tables(const uint8_t* mask, int Hq, int Hkv, int nQblk, int nKblk, int32_t* tables,
                    int32_t* counts, void* stream) {
  return ca_build_tables_batched(mask, 1, Hq, Hkv, nQblk, nKblk, tables, counts, stream);
}

int ca_build_tables_bits(const uint32_t* mask_bits, int nb, int Hq, int Hkv, int nQblk,
                         int nKblk, int32_t* tables, int32_t* counts, void* stream) {
  if (!mask_bits || !tables || !counts) return fail(CA_ERR_ARG, "ca_build_tables_bits: null pointer");
  if (nb < 1 || nb > 65535)
    return fail(CA_ERR_ARG, "ca_build_tables_bits: nb=%d out of [1,65535]", nb);
  if (Hq < 1 || Hkv < 1 || Hkv > Hq || Hq % Hkv || Hkv > 65535)
    return fail(CA_ERR_ARG, "ca_build_tables_bits: Hq=%d must be a positive multiple of Hkv=%d",
                Hq, Hkv);
  if (nQblk < 1) return fail(CA_ERR_ARG, "ca_build_tables_bits: nQblk=%d < 1", nQblk);
  if (nKblk < 1 || nKblk > 65536)
    return fail(CA_ERR_ARG, "ca_build_tables_bits: nKblk=%d out of [1,65536]", nKblk);
  if (reinterpret_cast<uintptr_t>(mask_bits) & 3u)
    return fail(CA_ERR_ARG, "ca_build_tables_bits: mask_bits must be 4-byte aligned");
  cudaError_t e = launch_build_tables_bits(mask_bits, nb, Hq, Hkv, nQblk, nKblk, tables, counts,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "ca_build_tables_bits launch");
  return CA_OK;
}

size_t ca_workspace_size(int dtype, int Hq, int Hkv, int head_dim, int block, int chunk_len,
                         int prefix_len, int num_pages, int n_splits) {
  Plan pl;
  SeqDesc d;
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32) return (size_t)-1;
  if (!plan(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d,
            dtype == CA_DTYPE_BF16))
    return (size_t)-1;
  if (num_pages < d.nKblk) return (size_t)-1;
  return ws_layout(dtype, Hq, Hkv, head_dim, block, chunk_len, num_pages, pl).total;
}

size_t ca_workspace_size_varlen(int dtype, int Hq, int Hkv, int head_dim, int block, int num_seqs,
                                int total_q, int max_kv_len, int num_pages, int n_splits) {
  Plan pl;
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32) return (size_t)-1;
  if (num_seqs < 1 || total_q < 0 || max_kv_len < 0 || num_pages < 1) return (size_t)-1;
  if (!plan_varlen(Hq, Hkv, head_dim, block, dtype, num_seqs, total_q, max_kv_len, n_splits, pl))
    return (size_t)-1;
  return ws_layout(dtype, Hq, Hkv, head_dim, block, total_q, num_pages, pl, num_seqs).total;
}

namespace {

// Shared tail of the attention entry points: fp32 casts, tensor maps, launch,
// merges.  `p` arrives with the sequence fields set; rows = rows of Q / O.
int run_attention(const char* who, const void* Q, const void* K_pages, const void* V_pages,
                  int dtype, int num_pages, int Hq, int Hkv, int D, int B, int rows,
                  const Plan& pl, const WsLayout& wl, uint8_t* ws, int grid, AttnParams& p,
                  cudaStream_t st) {
  const bool kv8 = dtype == CA_DTYPE_E4M3;  // Q is then already the f16 copy
  EncodeTiledFn enc = encoder();
  if (!enc) return fail(CA_ERR_LAUNCH, "%s: cuTensorMapEncodeTiled unavailable", who);
  const void* q = Q;
  const void* qlo = Q;
  const void* kp = K_pages;
  const void* vp = V_pages;
  cudaError_t e;
  if (dtype == CA_DTYPE_FP32) {
    // The tensor-core path is bf16 in, fp32 accumulate.  Q is kept as two
    // bf16 terms (its rounding error would shift every score of a row the
    // same way); K and V are rounded once.
    e = launch_split_f32_bf16(static_cast<const float*>(Q), ws + wl.q, ws + wl.qlo,
                              (size_t)rows * Hq * D, st);
    if (e == cudaSuccess)
      e = launch_cast_f32_bf16(static_cast<const float*>(K_pages), ws + wl.k,
                               (size_t)num_pages * Hkv * B * D, st);
    if (e == cudaSuccess)
      e = launch_cast_f32_bf16(static_cast<const float*>(V_pages), ws + wl.v,
                               (size_t)num_pages * Hkv * B * D, st);
    if (e != cudaSuccess) return cuda_fail(e, "cast to bf16");
    q = ws + wl.q;
    qlo = ws + wl.qlo;
    kp = ws + wl.k;
    vp = ws + wl.v;
  }

  CUtensorMap tq, tqlo, tk, tv;
  for (int which = 0; which < 2; ++which) {
    // rows beyond the last are zero-filled by the copy engine (a ragged last span)
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)std::max(rows, 1)};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(which ? &tqlo : &tq,
                     kv8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void*>(which ? qlo : q), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CA_ERR_LAUNCH, "%s: tensor map (Q) encode failed: %d", who, (int)r);
  }
  for (int which = 0; which < 2; ++which) {
    // bf16 pages: 64-element boxes with the 128-byte swizzle the MMAs read;
    // E4M3 pages: whole rows of D bytes, unswizzled, into the staging area
    const int esz = kv8 ? 1 : 2;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)B, (cuuint64_t)Hkv, (cuuint64_t)num_pages};
    cuuint64_t strides[3] = {(cuuint64_t)D * esz, (cuuint64_t)B * D * esz,
                             (cuuint64_t)Hkv * B * D * esz};
    // (the pair kernel loads K as 64-row halves of a stage)
    const cuuint32_t rows = (pl.pair && which == 0) ? 64u : (cuuint32_t)B;
    cuuint32_t box[4] = {kv8 ? (cuuint32_t)D : 64u, rows, 1, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(which ? &tv : &tk,
                     kv8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                     const_cast<void*>(which ? vp : kp), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     kv8 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(CA_ERR_LAUNCH, "%s: tensor map (%s pages) encode failed: %d", who,
                  which ? "V" : "K", (int)r);
  }

  p.tail_start = pl.tail_start;
  p.tail_k = pl.tail_k;
  p.n_tail = pl.n_tail;
  p.Otail = pl.tail_k > 1 ? reinterpret_cast<float*>(ws + wl.otail) : nullptr;
  p.LSEtail = pl.tail_k > 1 ? reinterpret_cast<float*>(ws + wl.lsetail) : nullptr;
  p.Opart = pl.n_splits > 1 ? reinterpret_cast<float*>(ws + wl.opart) : nullptr;
  p.LSEpart = pl.n_splits > 1 ? reinterpret_cast<float*>(ws + wl.lsepart) : nullptr;
  p.persistent = pl.persistent;
  p.n_units = pl.units;
  p.sk_ctas = pl.sk_ctas;
  p.sk_sched = pl.persistent ? reinterpret_cast<int32_t*>(ws + wl.sched) : nullptr;
  p.Osk = pl.persistent ? reinterpret_cast<float*>(ws + wl.osk) : nullptr;
  p.LSEsk = pl.persistent ? reinterpret_cast<float*>(ws + wl.lsesk) : nullptr;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = pl.G;
  p.HPU = pl.HPU;
  p.nhalves = pl.nhalves;
  p.L = rows;
  p.B = B;
  p.num_pages = num_pages;
  p.n_splits = pl.n_splits;
  p.out_f32 = dtype == CA_DTYPE_FP32 ? 1 : 0;  // E4M3 pages: O is bf16
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.wait_ns = kWaitNs;
  if (pl.pair)
    e = launch_chunk_attention_pair(tq, tk, tv, p, D, grid, st);
  else if (pl.tile)
    e = launch_chunk_attention_tile(tq, tk, tv, p, D, grid, st);
  else
    e = launch_chunk_attention(tq, tqlo, tk, tv, p, D, pl.NT, dtype == CA_DTYPE_FP32, kv8, grid,
                               st);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  if (pl.persistent) {
    e = launch_sk_combine(p, D, pl.NT, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention combine launch");
  }
  if (pl.n_splits > 1) {
    e = launch_split_combine(p.Opart, p.LSEpart, pl.n_splits, rows, Hq, D, p.O, p.LSE, p.out_f32, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention combine launch");
  }
  return CA_OK;
}

}  // namespace

int ca_chunk_attention(const void* Q, const void* K_pages, const void* V_pages, int dtype,
                       int num_pages, const int32_t* page_table, const int32_t* tables,
                       const int32_t* counts, int Hq, int Hkv, int head_dim, int block,
                       int chunk_len, int prefix_len, void* O, float* LSE, void* workspace,
                       size_t ws_bytes, int n_splits, int32_t* err_flag, void* stream) {
  if (!Q || !K_pages || !V_pages || !page_table || !tables || !counts || !O || !LSE)
    return fail(CA_ERR_ARG, "ca_chunk_attention: null pointer");
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32)
    return fail(CA_ERR_DTYPE, "ca_chunk_attention: dtype code %d not supported", dtype);
  if (block != 64 && block != 128)
    return fail(CA_ERR_ARG, "ca_chunk_attention: block=%d must be 64 or 128", block);
  Plan pl;
  SeqDesc d;
  if (!plan(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d,
            dtype == CA_DTYPE_BF16))
    return fail(CA_ERR_ARG,
                "ca_chunk_attention: unsupported shape Hq=%d Hkv=%d head_dim=%d block=%d "
                "chunk_len=%d prefix_len=%d",
                Hq, Hkv, head_dim, block, chunk_len, prefix_len);
  if (num_pages < d.nKblk)
    return fail(CA_ERR_ARG, "ca_chunk_attention: num_pages=%d < nKblk=%d", num_pages, d.nKblk);
  if (!aligned16(Q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(O))
    return fail(CA_ERR_ARG, "ca_chunk_attention: Q, K_pages, V_pages and O must be 16-byte aligned");
  const WsLayout wl = ws_layout(dtype, Hq, Hkv, head_dim, block, chunk_len, num_pages, pl);
  if (wl.total > 0 && (!workspace || ws_bytes < wl.total || !aligned16(workspace)))
    return fail(CA_ERR_WORKSPACE, "ca_chunk_attention: workspace of %zu bytes needed, got %zu",
                wl.total, workspace ? ws_bytes : (size_t)0);
  AttnParams p{};
  p.page_table = page_table;
  p.tables = tables;
  p.counts = counts;
  p.O = O;
  p.LSE = LSE;
  p.err = err_flag;
  p.n_units_dev = nullptr;
  p.seqs = nullptr;
  p.seq0 = d;
  p.num_seqs = 1;
  // When the prefix dominates, every span of a group sees nearly the same
  // blocks and costs the same: run the units group by group, so that the pages
  // in flight at one time are those of a few groups and stay in L2 for all the
  // spans that read them.  Otherwise later spans (more blocks) go first.
  p.unit_order = (pl.tile && (long long)prefix_len >= 2LL * chunk_len) ? 1 : 0;
  const int grid = plan_grid(pl);
  return run_attention("ca_chunk_attention", Q, K_pages, V_pages, dtype, num_pages, Hq, Hkv,
                       head_dim, block, chunk_len, pl, wl, static_cast<uint8_t*>(workspace), grid,
                       p, static_cast<cudaStream_t>(stream));
}

namespace {
// Fused and E4M3 calls: one CTA per unit (no persistent grid), KV splits when
// the units do not fill the SMs.
// pair_ok: the CTA-pair kernel may take the call (bf16, fused tables); it does
// when its shape rules hold (head_dim 128, an even number of head pairs).
bool plan_masked(int Hq, int Hkv, int head_dim, int block, int chunk_len, int prefix_len,
                 int n_splits, Plan& pl, SeqDesc& d, int max_nKblk = 2048, bool pair_ok = false) {
  if (pair_ok && plan(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d, true) &&
      pl.pair)
    return d.nKblk <= max_nKblk;
  if (!plan(Hq, Hkv, head_dim, block, chunk_len, prefix_len, 1, pl, d)) return false;
  if (d.nKblk > max_nKblk) return false;
  const int max_stages = (d.nKblk + pl.spb - 1) / pl.spb;
  int S = n_splits;
  const int sms = num_sms();
  if (S <= 0) S = pl.units >= sms ? 1 : (2 * sms + pl.units - 1) / pl.units;
  if (S > 16 && n_splits <= 0) S = 16;
  return plan_mode(pl, pl.units, max_stages, S, false);
}
}  // namespace

size_t ca_workspace_size_masked(int dtype, int Hq, int Hkv, int head_dim, int block,
                                int chunk_len, int prefix_len, int num_pages, int n_splits) {
  Plan pl;
  SeqDesc d;
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32) return (size_t)-1;
  if (!plan_masked(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d, 2048,
                   dtype == CA_DTYPE_BF16))
    return (size_t)-1;
  if (num_pages < d.nKblk) return (size_t)-1;
  return ws_layout(dtype, Hq, Hkv, head_dim, block, chunk_len, num_pages, pl).total;
}

int ca_chunk_attention_masked(const void* Q, const void* K_pages, const void* V_pages, int dtype,
                              int num_pages, const int32_t* page_table, const uint32_t* mask_bits,
                              int Hq, int Hkv, int head_dim, int block, int chunk_len,
                              int prefix_len, int32_t* tables_out, int32_t* counts_out, void* O,
                              float* LSE, void* workspace, size_t ws_bytes, int n_splits,
                              int32_t* err_flag, void* stream) {
  const char* who = "ca_chunk_attention_masked";
  if (!Q || !K_pages || !V_pages || !page_table || !mask_bits || !O || !LSE)
    return fail(CA_ERR_ARG, "%s: null pointer", who);
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32)
    return fail(CA_ERR_DTYPE, "%s: dtype code %d not supported", who, dtype);
  Plan pl;
  SeqDesc d;
  if (!plan_masked(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d, 2048,
                   dtype == CA_DTYPE_BF16))
    return fail(CA_ERR_ARG,
                "%s: unsupported shape Hq=%d Hkv=%d head_dim=%d block=%d chunk_len=%d "
                "prefix_len=%d (nKblk <= 2048)",
                who, Hq, Hkv, head_dim, block, chunk_len, prefix_len);
  if (num_pages < d.nKblk)
    return fail(CA_ERR_ARG, "%s: num_pages=%d < nKblk=%d", who, num_pages, d.nKblk);
  if (!aligned16(Q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(O))
    return fail(CA_ERR_ARG, "%s: Q, K_pages, V_pages and O must be 16-byte aligned", who);
  if (reinterpret_cast<uintptr_t>(mask_bits) & 3u)
    return fail(CA_ERR_ARG, "%s: mask_bits must be 4-byte aligned", who);
  const WsLayout wl = ws_layout(dtype, Hq, Hkv, head_dim, block, chunk_len, num_pages, pl);
  if (wl.total > 0 && (!workspace || ws_bytes < wl.total || !aligned16(workspace)))
    return fail(CA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, got %zu", who, wl.total,
                workspace ? ws_bytes : (size_t)0);
  AttnParams p{};
  p.page_table = page_table;
  p.O = O;
  p.LSE = LSE;
  p.err = err_flag;
  p.mask_bits = mask_bits;
  p.mask_words = (d.nKblk + 31) / 32;
  p.nQblk_mask = (chunk_len + block - 1) / block;
  p.tables_out = tables_out;
  p.counts_out = counts_out;
  p.seq0 = d;
  p.num_seqs = 1;
  p.unit_order = (pl.tile && (long long)prefix_len >= 2LL * chunk_len) ? 1 : 0;
  return run_attention(who, Q, K_pages, V_pages, dtype, num_pages, Hq, Hkv, head_dim, block,
                       chunk_len, pl, wl, static_cast<uint8_t*>(workspace), plan_grid(pl), p,
                       static_cast<cudaStream_t>(stream));
}

size_t ca_workspace_size_fp8(int Hq, int Hkv, int head_dim, int block, int chunk_len,
                             int prefix_len, int num_pages, int n_splits) {
  Plan pl;
  SeqDesc d;
  if (!plan_masked(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d, 1 << 30))
    return (size_t)-1;
  if (num_pages < d.nKblk) return (size_t)-1;
  return ws_layout(CA_DTYPE_E4M3, Hq, Hkv, head_dim, block, chunk_len, num_pages, pl, 0, d.nKblk)
      .total;
}

int ca_chunk_attention_fp8(const void* Q, const uint8_t* K_pages, const uint8_t* V_pages,
                           const float* K_scale, const float* V_scale, int num_pages,
                           const int32_t* page_table, const int32_t* tables,
                           const int32_t* counts, int Hq, int Hkv, int head_dim, int block,
                           int chunk_len, int prefix_len, void* O, float* LSE, void* workspace,
                           size_t ws_bytes, int n_splits, int32_t* err_flag, void* stream) {
  const char* who = "ca_chunk_attention_fp8";
  if (!Q || !K_pages || !V_pages || !K_scale || !V_scale || !page_table || !tables || !counts ||
      !O || !LSE)
    return fail(CA_ERR_ARG, "%s: null pointer", who);
  Plan pl;
  SeqDesc d;
  if (!plan_masked(Hq, Hkv, head_dim, block, chunk_len, prefix_len, n_splits, pl, d, 1 << 30))
    return fail(CA_ERR_ARG,
                "%s: unsupported shape Hq=%d Hkv=%d head_dim=%d block=%d chunk_len=%d "
                "prefix_len=%d",
                who, Hq, Hkv, head_dim, block, chunk_len, prefix_len);
  if (num_pages < d.nKblk)
    return fail(CA_ERR_ARG, "%s: num_pages=%d < nKblk=%d", who, num_pages, d.nKblk);
  if (!aligned16(Q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(O))
    return fail(CA_ERR_ARG, "%s: Q, K_pages, V_pages and O must be 16-byte aligned", who);
  const WsLayout wl =
      ws_layout(CA_DTYPE_E4M3, Hq, Hkv, head_dim, block, chunk_len, num_pages, pl, 0, d.nKblk);
  if (!workspace || ws_bytes < wl.total || !aligned16(workspace))
    return fail(CA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, got %zu", who, wl.total,
                workspace ? ws_bytes : (size_t)0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = launch_cast_bf16_f16(Q, ws + wl.q16, (size_t)chunk_len * Hq * head_dim, st);
  if (e == cudaSuccess)
    e = launch_gather_scales(tables, counts, page_table, K_scale, V_scale, Hkv, d.nKblk,
                             num_pages, reinterpret_cast<float2*>(ws + wl.esc), err_flag, st);
  if (e != cudaSuccess) return cuda_fail(e, "ca_chunk_attention_fp8 prologue launch");
  AttnParams p{};
  p.page_table = page_table;
  p.tables = tables;
  p.counts = counts;
  p.O = O;
  p.LSE = LSE;
  p.err = err_flag;
  p.escale = reinterpret_cast<const float2*>(ws + wl.esc);
  p.seq0 = d;
  p.num_seqs = 1;
  return run_attention(who, ws + wl.q16, K_pages, V_pages, CA_DTYPE_E4M3, num_pages, Hq, Hkv,
                       head_dim, block, chunk_len, pl, wl, ws, pl.units * pl.n_splits, p, st);
}

int ca_chunk_attention_varlen(const void* Q, const void* K_pages, const void* V_pages, int dtype,
                              int num_pages, int num_seqs, int total_q, const int32_t* cu_q,
                              const int32_t* prefix_len, int max_kv_len,
                              const int32_t* page_table, const int32_t* cu_pages,
                              const int32_t* tables, const int32_t* counts, int Hq, int Hkv,
                              int head_dim, int block, void* O, float* LSE, void* workspace,
                              size_t ws_bytes, int n_splits, int32_t* err_flag, void* stream) {
  const char* who = "ca_chunk_attention_varlen";
  if (!Q || !K_pages || !V_pages || !cu_q || !prefix_len || !page_table || !cu_pages ||
      !tables || !counts || !O || !LSE)
    return fail(CA_ERR_ARG, "%s: null pointer", who);
  if (dtype != CA_DTYPE_BF16 && dtype != CA_DTYPE_FP32)
    return fail(CA_ERR_DTYPE, "%s: dtype code %d not supported", who, dtype);
  if (num_seqs < 1 || total_q < 0 || max_kv_len < 0 || num_pages < 1)
    return fail(CA_ERR_ARG, "%s: num_seqs=%d total_q=%d max_kv_len=%d num_pages=%d", who,
                num_seqs, total_q, max_kv_len, num_pages);
  Plan pl;
  if (!plan_heads(Hq, Hkv, head_dim, block, pl))
    return fail(CA_ERR_ARG, "%s: unsupported shape Hq=%d Hkv=%d head_dim=%d block=%d", who, Hq,
                Hkv, head_dim, block);
  if (!plan_varlen(Hq, Hkv, head_dim, block, dtype, num_seqs, total_q, max_kv_len, n_splits, pl))
    return fail(CA_ERR_ARG, "%s: too many work units", who);
  if (!aligned16(Q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(O))
    return fail(CA_ERR_ARG, "%s: Q, K_pages, V_pages and O must be 16-byte aligned", who);
  const WsLayout wl = ws_layout(dtype, Hq, Hkv, head_dim, block, total_q, num_pages, pl, num_seqs);
  if (!workspace || ws_bytes < wl.total || !aligned16(workspace))
    return fail(CA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, got %zu", who, wl.total,
                workspace ? ws_bytes : (size_t)0);
  if (total_q == 0) return CA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  SeqDesc* seqs = reinterpret_cast<SeqDesc*>(ws + wl.seqs);
  int32_t* n_units = reinterpret_cast<int32_t*>(ws + wl.nunits);
  cudaError_t e = launch_varlen_setup(cu_q, prefix_len, cu_pages, num_seqs, total_q, block, Hkv,
                                      pl.nhalves, seqs, n_units, err_flag, st);
  if (e != cudaSuccess) return cuda_fail(e, "ca_chunk_attention_varlen setup launch");
  AttnParams p{};
  p.page_table = page_table;
  p.tables = tables;
  p.counts = counts;
  p.O = O;
  p.LSE = LSE;
  p.err = err_flag;
  p.n_units_dev = n_units;
  p.seqs = seqs;
  p.seq0 = SeqDesc{};
  p.num_seqs = num_seqs;
  const int grid = plan_grid(pl);
  return run_attention(who, Q, K_pages, V_pages, dtype, num_pages, Hq, Hkv, head_dim, block,
                       total_q, pl, wl, ws, grid, p, st);
}

int ca_check(int32_t* err_flag, void* stream) {
  if (!err_flag) return fail(CA_ERR_ARG, "ca_check: null err_flag");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, err_flag, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(err_flag, 0, sizeof(int32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "ca_check");
  if (h & CA_FLAG_TIMEOUT) return fail(CA_ERR_TIMEOUT, "device: a pipeline wait timed out");
  if (h & CA_FLAG_BOUNDS)
    return fail(CA_ERR_BOUNDS, "device: table entry, count or page id out of range");
  return CA_OK;
}

int ca_wait_probe(int32_t* err_flag, int limit_us, void* stream) {
  if (!err_flag || limit_us < 1 || limit_us > 10000000)
    return fail(CA_ERR_ARG, "ca_wait_probe: need err_flag and 1 <= limit_us <= 1e7");
  cudaError_t e =
      launch_wait_probe(err_flag, (unsigned long long)limit_us * 1000ull, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "ca_wait_probe launch");
  return CA_OK;
}

}  // extern "C"
