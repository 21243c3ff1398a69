// flashloop_gate_noalloc: the token change gate for callers that cannot
// allocate device memory.
//
// Some callers can't call cudaMalloc: a serving process that reserved all of
// HBM for its cache pools at start-up and runs with a frozen budget, a host
// framework that owns every device allocation, or a latency-critical path
// where cudaMalloc's implicit device synchronisation (or its failure under
// memory pressure) is not acceptable.  Such callers may also have no
// workspace to lend.  This entry point runs the same gate kernel as
// flashloop_gate, but its scratch (one decision byte per candidate plus the
// compaction ticket) lives in a file-scope device array that the library
// owns: every GPU that loads the library holds those 64 KiB + 256 bytes
// until the process exits.  The caller still passes inputs and outputs.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace fl {

// Same kernel as flashloop_gate (defined in gate.cu).
__global__ void gate_kernel(const uint16_t* __restrict__ x_cur, const uint16_t* __restrict__ x_prev,
                            int S, int d, const int32_t* __restrict__ prev_active,
                            const int32_t* __restrict__ n_prev_ptr, int prev_cap, float tau2,
                            uint8_t* __restrict__ flags, unsigned int* __restrict__ ticket,
                            int32_t* __restrict__ active_out, int32_t* __restrict__ slot_out,
                            int32_t* __restrict__ n_out, int out_cap, int32_t* __restrict__ err);

// Parameter and architecture checks shared by every entry point (api.cu).
int check_params_and_arch(const flashloop_params* p);

constexpr int kNoallocThreads = 256;
constexpr size_t kNoallocTicketBytes = 256;

// The library-owned scratch: the ticket, then one flag per candidate.
static __device__ __align__(256) unsigned char g_gate_scratch[kNoallocTicketBytes +
                                                               FLASHLOOP_NOALLOC_MAX_CANDIDATES];

// Device address of g_gate_scratch, resolved once per device and context.
// In host code the symbol is only a host-side stand-in, so the address must
// come from cudaGetSymbolAddress with the device current.  The address is
// kept together with the context it was resolved in: after the caller
// destroys and re-creates the context (cudaDeviceReset, a new primary
// context) the module is loaded again, possibly elsewhere, and the address
// is looked up again instead of reusing a stale one.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

static CtxGetCurrentFn ctx_get_current() {
  static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return nullptr;
  }();
  return fn;
}

static CUcontext current_context() {
  CUcontext ctx = nullptr;
  const CtxGetCurrentFn fn = ctx_get_current();
  if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

struct ScratchAddr {
  CUcontext ctx;
  void* addr;
};
static std::mutex g_scratch_mutex;
static ScratchAddr g_scratch_addr[128];

static int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return FLASHLOOP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchAddr& c = g_scratch_addr[dev];
  const CUcontext ctx = current_context();
  if (c.addr == nullptr || ctx == nullptr || c.ctx != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_gate_scratch) != cudaSuccess || ptr == nullptr)
      return FLASHLOOP_ERR_CUDA;
    c.addr = ptr;
    c.ctx = current_context();  // the lookup may have made the primary context current
  }
  *out = c.addr;
  return FLASHLOOP_OK;
}

}  // namespace fl

extern "C" int flashloop_gate_noalloc(const flashloop_params* p, const uint16_t* x_cur,
                                      const uint16_t* x_prev, const int32_t* prev_active,
                                      const int32_t* n_prev, int32_t prev_capacity,
                                      int32_t* active_out, int32_t* slot_out,
                                      int32_t* n_active_out, int32_t out_capacity,
                                      int32_t* err_word, void* stream) {
  using namespace fl;
  // The same parameter, architecture and argument checks as flashloop_gate,
  // in the same order, so both refuse the same inputs with the same codes.
  int rc = check_params_and_arch(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (!x_cur || !x_prev || !active_out || !slot_out || !n_active_out) return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_active != nullptr && n_prev == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_capacity < 1 || prev_capacity > p->seq || out_capacity < 1 || out_capacity > p->seq)
    return FLASHLOOP_ERR_INVALID_ARG;
  // The scratch holds one byte per candidate: larger problems are refused.
  const int candidates = prev_active ? prev_capacity : p->seq;
  if (candidates > FLASHLOOP_NOALLOC_MAX_CANDIDATES) return FLASHLOOP_ERR_UNSUPPORTED;
  void* base = nullptr;
  rc = scratch_address(&base);
  if (rc != FLASHLOOP_OK) return rc;
  unsigned int* ticket = static_cast<unsigned int*>(base);
  uint8_t* flags = static_cast<uint8_t*>(base) + kNoallocTicketBytes;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents; the ticket must start at zero.
  if (cudaMemsetAsync(ticket, 0, sizeof(unsigned int), s) != cudaSuccess) return FLASHLOOP_ERR_CUDA;
  const int rows_per_block = kNoallocThreads / 32;
  int grid = (prev_capacity + rows_per_block - 1) / rows_per_block;
  if (grid > 148 * 8) grid = 148 * 8;
  if (grid < 1) grid = 1;
  gate_kernel<<<grid, kNoallocThreads, 0, s>>>(x_cur, x_prev, p->seq, p->d_model, prev_active, n_prev,
                                               prev_capacity, p->tau * p->tau, flags, ticket,
                                               active_out, slot_out, n_active_out, out_capacity,
                                               err_word);
  return cudaGetLastError() == cudaSuccess ? FLASHLOOP_OK : FLASHLOOP_ERR_CUDA;
}
