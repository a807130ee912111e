// bsa_forward_noalloc: bsa_forward with its scratch memory built into the library.
//
// Some callers cannot call cudaMalloc at all: a host that hands every byte of device
// memory to its own pool and forbids allocations from plug-ins, a serving loop that must
// not take cudaMalloc's implicit device synchronisation, or an embedded runtime with a
// fixed memory budget decided at load time. For them this entry point takes the same
// inputs and outputs as bsa_forward but no workspace: the scratch (the validation flag
// and the bf16 copies of the PISA statistics) lives in one file-scope __device__ array
// of BSA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds until the
// process exits.
//
// The array's name is a host-side stand-in in host code, not a device address: every
// call looks up its device address on the current device with cudaGetSymbolAddress
// (cheap once the module is loaded; on the first call on a device it may load the
// module, which is why that first call must come before any stream capture). Looking it
// up on every call, rather than caching it, keeps the address valid across a
// cudaDeviceReset or a recreated primary context. All calls share the array and it
// keeps the last call's contents; the launch sequence clears the flag word it needs
// zeroed. Two calls whose kernels overlap on the GPU (different streams, or different
// host threads) race on the array.
#include "../../include/bsattn.h"
#include "internal.h"

namespace bsa {
namespace {

static __device__ __align__(256) unsigned char g_forward_scratch[BSA_NOALLOC_SCRATCH_BYTES];

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_forward_noalloc(const void* Q, const void* K, const void* V,
                                          int32_t Bt, int32_t H, int32_t L, int32_t d,
                                          int32_t block, const int32_t* key_valid,
                                          const int32_t* row_ptr,
                                          const int32_t* col_idx, int64_t nnz_total,
                                          int32_t csr_per_head, int32_t mode, const float* kbar,
                                          const float* vsum, const float* Hbar, float scale,
                                          void* O, float* lse, int32_t* status, void* stream) {
  bsa::ForwardArgs a = bsa::forward_args(Q, K, V, Bt, H, L, d, block, key_valid, row_ptr, col_idx,
                                         nnz_total, csr_per_head, mode, kbar, vsum, Hbar, scale,
                                         O, lse, nullptr, status);
  const bsa_status r = bsa::check_forward_args(a);
  if (r != BSA_OK) return r;
  // keep-or-drop and the per-block mode touch only the flag at the start of the scratch;
  // PISA needs all of it
  const size_t need = mode == BSA_MODE_PISA ? bsa::forward_workspace(a.s) : 256;
  if (need > (size_t)BSA_NOALLOC_SCRATCH_BYTES) return BSA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, bsa::g_forward_scratch) != cudaSuccess || scratch == nullptr)
    return BSA_ERR_CUDA;
  a.ws = scratch;
  return bsa::launch_forward(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? BSA_OK
             : BSA_ERR_CUDA;
}
