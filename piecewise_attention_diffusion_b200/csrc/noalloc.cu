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
// The array is a host-side stand-in in host code, not a device address: its device
// address is looked up once per device with cudaGetSymbolAddress (on the first call made
// with that device current) and cached. All calls share the array and it keeps the last
// call's contents; the launch sequence clears the flag word it needs zeroed. Two calls
// whose kernels overlap on the GPU (different streams, or different host threads) race
// on the array.
#include <mutex>

#include "../../include/bsattn.h"
#include "internal.h"

namespace bsa {
namespace {

static __device__ __align__(256) unsigned char g_forward_scratch[BSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_forward_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_forward_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
  const bsa::Shape s{Bt, H, L, d, block, key_valid};
  if (Bt <= 0 || H <= 0 || L <= 0 || d <= 0 || block <= 0) return BSA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (block != 64 && block != 128) || L % block != 0 ||
      s.M() > 2048 || (int64_t)Bt * H > 65535 || (int64_t)Bt * H * L * d >= (int64_t)1 << 40)
    return BSA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !O || !row_ptr) return BSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(key_valid) & 3u) != 0) return BSA_ERR_INVALID_ARG;
  if (nnz_total < 0 || (nnz_total > 0 && col_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  if (nnz_total >= INT32_MAX) return BSA_ERR_UNSUPPORTED;
  if (!bsa::aligned16(Q) || !bsa::aligned16(K) || !bsa::aligned16(V) || !bsa::aligned16(O))
    return BSA_ERR_INVALID_ARG;
  if (csr_per_head != 0 && csr_per_head != 1) return BSA_ERR_INVALID_ARG;
  if (mode != BSA_MODE_KEEP_OR_DROP && mode != BSA_MODE_PISA && mode != BSA_MODE_PISA_BLOCK)
    return BSA_ERR_INVALID_ARG;
  if (mode == BSA_MODE_PISA && (!kbar || !vsum || !Hbar)) return BSA_ERR_INVALID_ARG;
  if (!(scale >= 0.f)) return BSA_ERR_INVALID_ARG;
  // keep-or-drop and the per-block mode touch only the flag at the start of the scratch;
  // PISA needs all of it
  const size_t need = mode == BSA_MODE_PISA ? bsa::forward_workspace(s) : 256;
  if (need > (size_t)BSA_NOALLOC_SCRATCH_BYTES) return BSA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (bsa::scratch_address(&scratch) != cudaSuccess) return BSA_ERR_CUDA;
  bsa::ForwardArgs a;
  a.s = s;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.nnz_total = nnz_total;
  a.csr_per_head = csr_per_head;
  a.mode = mode;
  a.kbar = kbar;
  a.vsum = vsum;
  a.Hbar = Hbar;
  a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  a.O = O;
  a.lse = lse;
  a.ws = scratch;
  a.status = status;
  return bsa::launch_forward(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? BSA_OK
             : BSA_ERR_CUDA;
}
