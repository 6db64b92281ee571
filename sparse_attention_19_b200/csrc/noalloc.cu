// noalloc.cu -- dsa_sparse_attn_noalloc: dsa_sparse_attn whose split-k partials
// live in a fixed array of this library's device image instead of a workspace
// the caller allocates.
//
// The array sits in this translation unit alone, which holds no kernel: with the
// CUDA runtime's default lazy module loading, its DSA_NOALLOC_SCRATCH_BYTES of
// device memory are reserved on a device only once this entry point looks the
// array up there, not by every user of the library.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "dsa.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The driver's id of the context current on this thread (0 when none is current
// or the driver cannot say).  Ids are unique for the life of the process, so a
// context created after a reset never matches an earlier one.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the array in the current device's context.  In host code the
// array's name only stands for it; the address is looked up with that device
// current, once per device and context, and reused until the context changes
// (after cudaDeviceReset, say, the module is loaded again and may sit elsewhere).
dsa_status scratch_address(void** ptr) {
  struct Slot {
    unsigned long long ctx_id;
    void* addr;
  };
  static std::mutex mu;
  static Slot slots[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  Slot& s = slots[dev];
  const unsigned long long id = current_context_id();
  if (!s.addr || id == 0 || id != s.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
    s.addr = p;
    s.ctx_id = current_context_id();   // the lookup makes the primary context current if none was
  }
  *ptr = s.addr;
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_sparse_attn_noalloc(const dsa_attn_args* args, int B, int Lq, int Lk,
                                              const int32_t* indices, int k, void* out, float* lse,
                                              void* stream) {
  // Partials needed for these sizes (0 when no row is split, or when the
  // arguments are invalid, which dsa_sparse_attn then reports).
  const size_t need = args ? dsa_workspace_size(DSA_OP_SPARSE_ATTN, B, Lq, Lk, k, args->H, args->d_v) : 0;
  if (need > DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    const dsa_status s = scratch_address(&ws);
    if (s != DSA_OK) return s;
  }
  return dsa_sparse_attn(args, B, Lq, Lk, indices, k, out, lse, ws, need > 0 ? DSA_NOALLOC_SCRATCH_BYTES : 0,
                         stream);
}
