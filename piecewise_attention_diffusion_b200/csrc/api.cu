// C ABI of libbsattn: host-side argument validation, then asynchronous launches on the
// caller's stream. No call allocates, frees or synchronises.
#include <stdint.h>

#include "../../include/bsattn.h"
#include "internal.h"

namespace {

using bsa::Shape;

constexpr int kMaxBlocks = 2048;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by precompute / route / forward.
bsa_status check_shape(const Shape& s) {
  if (s.Bt <= 0 || s.H <= 0 || s.L <= 0 || s.d <= 0 || s.block <= 0)
    return BSA_ERR_INVALID_ARG;
  if (s.d != 64 && s.d != 128) return BSA_ERR_UNSUPPORTED;
  if (s.block != 64 && s.block != 128) return BSA_ERR_UNSUPPORTED;
  if (s.L % s.block != 0) return BSA_ERR_UNSUPPORTED;
  if (s.M() > kMaxBlocks) return BSA_ERR_UNSUPPORTED;
  if ((int64_t)s.Bt * s.H * s.L * s.d >= (int64_t)1 << 40) return BSA_ERR_UNSUPPORTED;
  if ((int64_t)s.Bt * s.H > 65535) return BSA_ERR_UNSUPPORTED;  // grid.y limit
  if ((reinterpret_cast<uintptr_t>(s.key_valid) & 3u) != 0) return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

bsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

bool workspace_ok(size_t need, const void* ws, size_t ws_bytes) {
  return need == 0 || (ws != nullptr && ws_bytes >= need && aligned16(ws));
}

int mask_blocks(const bsa_mask_desc* d) {
  if (d == nullptr) return -1;
  if (d->n_text_blocks < 0 || d->grid_h < 0 || d->grid_w < 0 || d->radius < 0 ||
      d->global_stride < 0)
    return -1;
  if ((d->grid_h == 0) != (d->grid_w == 0)) return -1;
  const int64_t m = (int64_t)d->n_text_blocks + (int64_t)d->grid_h * d->grid_w;
  if (m <= 0 || m > kMaxBlocks) return -1;
  return (int)m;
}

}  // namespace

namespace bsa {

float forward_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / sqrtf((float)d); }

ForwardArgs forward_args(const void* Q, const void* K, const void* V, int Bt, int H, int L, int d,
                         int block, const int32_t* key_valid, const int32_t* row_ptr,
                         const int32_t* col_idx, int64_t nnz_total, int csr_per_head, int mode,
                         const float* kbar, const float* vsum, const float* Hbar, float scale,
                         void* O, float* lse, void* ws, int32_t* status) {
  ForwardArgs a;
  a.s = Shape{Bt, H, L, d, block, key_valid};
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
  a.scale = scale;
  a.O = O;
  a.lse = lse;
  a.ws = ws;
  a.status = status;
  return a;
}

bsa_status check_forward_args(const ForwardArgs& a) {
  bsa_status r = check_shape(a.s);
  if (r != BSA_OK) return r;
  if (!a.Q || !a.K || !a.V || !a.O || !a.row_ptr) return BSA_ERR_INVALID_ARG;
  if (a.nnz_total < 0 || (a.nnz_total > 0 && a.col_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  if (a.nnz_total >= INT32_MAX) return BSA_ERR_UNSUPPORTED;
  if (!aligned16(a.Q) || !aligned16(a.K) || !aligned16(a.V) || !aligned16(a.O))
    return BSA_ERR_INVALID_ARG;
  if (a.csr_per_head != 0 && a.csr_per_head != 1) return BSA_ERR_INVALID_ARG;
  if (a.mode != BSA_MODE_KEEP_OR_DROP && a.mode != BSA_MODE_PISA &&
      a.mode != BSA_MODE_PISA_BLOCK)
    return BSA_ERR_INVALID_ARG;
  if (a.mode == BSA_MODE_PISA && (!a.kbar || !a.vsum || !a.Hbar)) return BSA_ERR_INVALID_ARG;
  if (!(a.scale >= 0.f)) return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

}  // namespace bsa

extern "C" {

int32_t bsa_version(void) { return 110; }

const char* bsa_status_string(int32_t code) {
  switch (code) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_BAD_CSR: return "BSA_ERR_BAD_CSR";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
    case BSA_ERR_CAPACITY: return "BSA_ERR_CAPACITY";
    case BSA_ERR_SCRATCH_LIMIT: return "BSA_ERR_SCRATCH_LIMIT";
    case BSA_ERR_BAD_PADDING: return "BSA_ERR_BAD_PADDING";
    default: return "BSA_UNKNOWN_STATUS";
  }
}

int32_t bsa_mask_blocks(const bsa_mask_desc* desc) { return mask_blocks(desc); }

size_t bsa_workspace_bytes(int32_t call, int32_t Bt, int32_t H, int32_t L, int32_t d,
                           int32_t block) {
  const Shape s{Bt, H, L, d, block};
  if (call == BSA_CALL_BUILD_MASK) return 0;
  if (check_shape(s) != BSA_OK) return 0;
  if (call == BSA_CALL_PRECOMPUTE) return bsa::precompute_workspace(s);
  if (call == BSA_CALL_ROUTE) return bsa::route_workspace(s);
  if (call == BSA_CALL_FORWARD) return bsa::forward_workspace(s);
  return 0;
}

bsa_status bsa_build_mask(const bsa_mask_desc* desc, int32_t* row_ptr, int32_t* col_idx,
                          int64_t col_capacity, int32_t* status, void* stream) {
  const int M = mask_blocks(desc);
  if (M < 0) return BSA_ERR_INVALID_ARG;
  if (row_ptr == nullptr || col_idx == nullptr || col_capacity < 0) return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_build_mask(*desc, M, row_ptr, col_idx, col_capacity, status,
                                          static_cast<cudaStream_t>(stream)));
}

bsa_status bsa_precompute(const void* K, const void* V, int32_t Bt, int32_t H, int32_t L,
                          int32_t d, int32_t block, const int32_t* key_valid, float* kbar,
                          float* vsum, float* Hbar, float* Mnorm, float* Hblk,
                          void* workspace, size_t ws_bytes, int32_t* status, void* stream) {
  const Shape s{Bt, H, L, d, block, key_valid};
  bsa_status r = check_shape(s);
  if (r != BSA_OK) return r;
  if (!K || !V || !kbar || !vsum || !Hbar || !Mnorm) return BSA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V)) return BSA_ERR_INVALID_ARG;
  if (!workspace_ok(bsa::precompute_workspace(s), workspace, ws_bytes)) return BSA_ERR_WORKSPACE;
  return from_cuda(bsa::launch_precompute(s, K, V, kbar, vsum, Hbar, Mnorm, Hblk, workspace,
                                          status, static_cast<cudaStream_t>(stream)));
}

bsa_status bsa_route(const void* Q, const float* kbar, const float* Mnorm, int32_t Bt,
                     int32_t H, int32_t L, int32_t d, int32_t block, const int32_t* key_valid,
                     int32_t k_top, float lambda, float scale, int32_t* row_ptr,
                     int32_t* col_idx, float* scores, void* workspace, size_t ws_bytes,
                     int32_t* status, void* stream) {
  const Shape s{Bt, H, L, d, block, key_valid};
  bsa_status r = check_shape(s);
  if (r != BSA_OK) return r;
  if (!Q || !kbar || !Mnorm || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
  if (!aligned16(Q)) return BSA_ERR_INVALID_ARG;
  if (k_top < 1 || k_top > s.M()) return BSA_ERR_INVALID_ARG;
  if ((int64_t)s.BH() * s.M() * k_top >= INT32_MAX) return BSA_ERR_UNSUPPORTED;
  if (!(lambda >= 0.f) || !(scale >= 0.f)) return BSA_ERR_INVALID_ARG;
  if (!workspace_ok(bsa::route_workspace(s), workspace, ws_bytes)) return BSA_ERR_WORKSPACE;
  const float sc = bsa::forward_scale(scale, d);
  return from_cuda(bsa::launch_route(s, Q, kbar, Mnorm, k_top, lambda, sc, row_ptr, col_idx,
                                     scores, workspace, status,
                                     static_cast<cudaStream_t>(stream)));
}

bsa_status bsa_forward(const void* Q, const void* K, const void* V, int32_t Bt, int32_t H,
                       int32_t L, int32_t d, int32_t block, const int32_t* key_valid,
                       const int32_t* row_ptr,
                       const int32_t* col_idx, int64_t nnz_total, int32_t csr_per_head,
                       int32_t mode, const float* kbar, const float* vsum,
                       const float* Hbar, float scale, void* O, float* lse,
                       void* workspace, size_t ws_bytes, int32_t* status, void* stream) {
  const bsa::ForwardArgs a = bsa::forward_args(Q, K, V, Bt, H, L, d, block, key_valid, row_ptr,
                                               col_idx, nnz_total, csr_per_head, mode, kbar,
                                               vsum, Hbar, scale, O, lse, workspace, status);
  const bsa_status r = bsa::check_forward_args(a);
  if (r != BSA_OK) return r;
  if (!workspace_ok(bsa::forward_workspace(a.s), workspace, ws_bytes)) return BSA_ERR_WORKSPACE;
  return from_cuda(bsa::launch_forward(a, static_cast<cudaStream_t>(stream)));
}

bsa_status bsa_selftest_forward_timeout(const void* Q, const void* K, const void* V, int32_t Bt,
                                        int32_t H, int32_t L, int32_t d, int32_t block,
                                        const int32_t* row_ptr, const int32_t* col_idx,
                                        int64_t nnz_total, int32_t mode, const float* kbar,
                                        const float* vsum, const float* Hbar, void* O,
                                        void* workspace, size_t ws_bytes, int64_t wait_ns,
                                        int32_t* status, void* stream) {
  if (status == nullptr || wait_ns < 1 || wait_ns > 10000000000ll) return BSA_ERR_INVALID_ARG;
  bsa::ForwardArgs a = bsa::forward_args(Q, K, V, Bt, H, L, d, block, nullptr, row_ptr, col_idx,
                                         nnz_total, 1, mode, kbar, vsum, Hbar, 0.f, O, nullptr,
                                         workspace, status);
  const bsa_status r = bsa::check_forward_args(a);
  if (r != BSA_OK) return r;
  if (!workspace_ok(bsa::forward_workspace(a.s), workspace, ws_bytes)) return BSA_ERR_WORKSPACE;
  a.wait_ns = static_cast<uint64_t>(wait_ns);
  return from_cuda(bsa::launch_forward(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
