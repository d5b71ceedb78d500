// noalloc.cu — ca_chunk_attention_noalloc: chunk attention for callers that
// must not allocate device memory.
//
// Some callers cannot call cudaMalloc on the path that runs attention: an
// inference engine that reserves the whole device up front and hands out
// memory only through its own allocator, or a latency-critical loop where an
// allocation (and the device-wide synchronisation it may imply) is not
// allowed.  ca_chunk_attention needs caller-provided workspace when it splits
// the KV range of each work unit; this entry point instead keeps the split
// partials in a fixed scratch array compiled into the library, so the caller
// passes only inputs and outputs.
//
// The scratch array lives in this file.  Every GPU that loads the library
// holds kNoAllocScratchBytes of device memory for it until the process exits.
// All calls on a device share the one array and it keeps the contents of the
// last call; nothing in it has to start at zero (every partial a split reads
// was written by the same call).  Calls whose kernels overlap on the GPU —
// on two streams, or from two host threads — race on the array and give
// wrong results: serialise them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "compactattn.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;

// Per device: the unique id of the context the address was looked up in, and
// the address.  A reset of the device (cudaDeviceReset) destroys the context
// and the next one reloads the module, so the array may then sit at another
// address; a cached address is only reused while the device's current context
// is the one it came from.  Context ids (cuCtxGetId) are never reused within a
// process, unlike context handles.
struct ScratchAddr {
  unsigned long long ctx_id = 0;
  bool valid = false;
  void* ptr = nullptr;
};
ScratchAddr g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

void* driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return p;
  return nullptr;
}

// Unique id of the calling thread's current context; false if there is none.
bool current_ctx_id(unsigned long long* id) {
  static std::once_flag once;
  static CtxGetCurrentFn get = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    get = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
    get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  });
  CUcontext ctx = nullptr;
  if (!get || !get_id || get(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current device's current
// context.  In host code the array's name only stands in for the symbol; the
// kernels need the address cudaGetSymbolAddress returns for this device.  The
// lookup runs on the first call per device and again on the first call after
// that device's context has changed (a reset).
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    ca::set_last_error("ca_chunk_attention_noalloc: no usable current device");
    return CA_ERR_LAUNCH;
  }
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchAddr& c = g_scratch[dev];
  if (!have_id || !c.valid || c.ctx_id != id) {
    // (the lookup also binds the device's primary context to this thread when
    // no context is current yet; the context is read again after it)
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      ca::set_last_error("ca_chunk_attention_noalloc: cudaGetSymbolAddress of the scratch failed");
      return CA_ERR_LAUNCH;
    }
    if (!current_ctx_id(&id)) {
      ca::set_last_error("ca_chunk_attention_noalloc: cannot identify the current CUDA context");
      return CA_ERR_LAUNCH;
    }
    c.ctx_id = id;
    c.valid = true;
    c.ptr = p;
  }
  *out = c.ptr;
  return CA_OK;
}

}  // namespace

extern "C" {

size_t ca_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int ca_chunk_attention_noalloc(const void* Q, const void* K_pages, const void* V_pages,
                               int num_pages, const int32_t* page_table, const int32_t* tables,
                               const int32_t* counts, int Hq, int Hkv, int head_dim, int block,
                               int chunk_len, int prefix_len, void* O, float* LSE, int n_splits,
                               int32_t* err_flag, void* stream) {
  const size_t need = ca_workspace_size(CA_DTYPE_BF16, Hq, Hkv, head_dim, block, chunk_len,
                                        prefix_len, num_pages, n_splits);
  if (need == (size_t)-1)
    return ca_chunk_attention(Q, K_pages, V_pages, CA_DTYPE_BF16, num_pages, page_table, tables,
                              counts, Hq, Hkv, head_dim, block, chunk_len, prefix_len, O, LSE,
                              nullptr, 0, n_splits, err_flag, stream);  // reports the bad shape
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "ca_chunk_attention_noalloc: these shapes need %zu bytes of split scratch, more "
             "than the library's fixed %zu bytes; use fewer splits or ca_chunk_attention",
             need, kNoAllocScratchBytes);
    ca::set_last_error(msg);
    return CA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    const int rc = scratch_address(&scratch);
    if (rc != CA_OK) return rc;
  }
  return ca_chunk_attention(Q, K_pages, V_pages, CA_DTYPE_BF16, num_pages, page_table, tables,
                            counts, Hq, Hkv, head_dim, block, chunk_len, prefix_len, O, LSE,
                            scratch, need > 0 ? kNoAllocScratchBytes : 0, n_splits, err_flag,
                            stream);
}

}  // extern "C"
