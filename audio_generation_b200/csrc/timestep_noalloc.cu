// h3_timestep_modulation_noalloc: the timestep-modulation prologue for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or hand the library a scratch buffer)
// at the point where they compute the per-forward modulation: a serving loop
// whose device memory is reserved up front by its own pool and that forbids
// further device allocations, or a latency-critical loop (an audio/video frame
// callback) in which allocation is not allowed. This entry point computes the
// same result as h3_timestep_modulation with its scratch (sinusoid, MLP hidden
// and time-embedding rows) in a fixed, statically sized device array that
// belongs to the library; the caller passes only inputs and outputs.
//
// Limits and sharing:
//  - The array holds kStaticScratchBytes (4 MiB); n_t is accepted only while
//    the scratch of the CUDA-core form of the prologue fits in it (at the full
//    constructor widths, n_t <= 126). Larger requests return H3_ERR_WORKSPACE
//    before any work is queued. (h3_timestep_modulation switches to
//    tensor-core GEMMs over split operands from 65 timesteps on; this entry
//    does not.)
//  - Every GPU that loads the library holds its own copy of the array until the
//    process exits.
//  - All calls on a device share that one array, and the array keeps the last
//    call's contents. Nothing in it needs to start at zero (every scratch value
//    is written before it is read), but calls whose work overlaps on the GPU
//    (different streams without ordering between them) race on it: order them
//    on one stream or with events.
//  - The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current); make that first call
//    before any stream capture. The address is looked up again when the
//    device's context has changed since (after a cudaDeviceReset).
#include "internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;

// File-scope device scratch. In host code this name is only a stand-in for the
// symbol, never a usable address: kernels receive the device address obtained
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_timestep_scratch[kStaticScratchBytes];

// The array's device address, looked up with the device current on the first
// call on that device, and again if the device's context has been replaced
// since (cudaDeviceReset loads the module anew, possibly at another address).
h3::SymbolAddressCache g_scratch_cache;

cudaError_t lookup_scratch(void** p) { return cudaGetSymbolAddress(p, g_timestep_scratch); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" h3_status h3_timestep_modulation_noalloc(const h3_dims* dims, int n_t, const float* t,
                                                    const float* w_t1, const float* w_t2,
                                                    const float* w_proj, float* tmod,
                                                    h3_stream_t stream) {
  // Same checks, in the same order, as h3_timestep_modulation.
  const h3_status dims_ok = h3::check_dims(dims);
  if (dims_ok != H3_OK) return dims_ok;
  if (n_t < 0) return H3_ERR_ARG;
  // This entry always runs the CUDA-core form of the prologue GEMMs (the split
  // form's operand copies would not fit the fixed array).
  const size_t need = h3::timestep_workspace_bytes(*dims, n_t, false);
  if (need > kStaticScratchBytes) return H3_ERR_WORKSPACE;
  if (n_t == 0) return H3_OK;
  if (!t || !w_t1 || !w_t2 || !w_proj || !tmod) return H3_ERR_ARG;
  if (!aligned16(t) || !aligned16(w_t1) || !aligned16(w_t2) || !aligned16(w_proj) ||
      !aligned16(tmod))
    return H3_ERR_ALIGN;
  void* scratch = nullptr;
  const h3_status s = h3::symbol_address(g_scratch_cache, lookup_scratch, &scratch);
  if (s != H3_OK) return s;
  const cudaError_t e = h3::launch_timestep(*dims, n_t, t, w_t1, w_t2, w_proj, tmod, scratch,
                                            false, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? H3_OK : H3_ERR_CUDA;
}
