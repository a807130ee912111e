// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bsattn.h"

namespace bsa {

struct Shape {
  int Bt, H, L, d, block;
  const int32_t* key_valid = nullptr;  // real tokens per block (device int32 [M]), or null
  int BH() const { return Bt * H; }
  int M() const { return L / block; }
};

// Workspace size of each call (bytes); 0 if none.
size_t precompute_workspace(const Shape& s);
size_t forward_workspace(const Shape& s);

cudaError_t launch_build_mask(const bsa_mask_desc& desc, int M, int32_t* row_ptr,
                              int32_t* col_idx, int64_t cap, int32_t* status,
                              cudaStream_t st);

cudaError_t launch_precompute(const Shape& s, const void* K, const void* V, float* kbar,
                              float* vsum, float* Hbar, float* Mnorm, float* Hblk,
                              void* ws, int32_t* status, cudaStream_t st);

// Routing workspace: the column sums of every 32-row segment of Q (fp32 [BH, L/32, d]).
size_t route_workspace(const Shape& s);

cudaError_t launch_route(const Shape& s, const void* Q, const float* kbar,
                         const float* Mnorm, int k_top, float lambda, float scale,
                         int32_t* row_ptr, int32_t* col_idx, float* scores, void* ws,
                         int32_t* status, cudaStream_t st);

struct ForwardArgs {
  Shape s;
  const void *Q, *K, *V;
  const int32_t *row_ptr, *col_idx;
  int64_t nnz_total;
  int csr_per_head;
  int mode;
  const float *kbar, *vsum, *Hbar;
  float scale;
  void* O;
  float* lse;
  void* ws;
  int32_t* status;
  uint64_t wait_ns = 0;  // limit of the attention kernel's bounded waits; 0: the default
};

// bsa_forward's arguments as one record (the scale as given; 0 is resolved at launch).
ForwardArgs forward_args(const void* Q, const void* K, const void* V, int Bt, int H, int L, int d,
                         int block, const int32_t* key_valid, const int32_t* row_ptr,
                         const int32_t* col_idx, int64_t nnz_total, int csr_per_head, int mode,
                         const float* kbar, const float* vsum, const float* Hbar, float scale,
                         void* O, float* lse, void* ws, int32_t* status);

// Host-side checks of bsa_forward's arguments, all but the workspace: shapes, pointers,
// alignment, list sizes, mode, scale. BSA_OK or the status to return.
bsa_status check_forward_args(const ForwardArgs& a);

// The scale a forward call uses: `scale`, or 1/sqrt(d) when it is 0.
float forward_scale(float scale, int d);

cudaError_t launch_forward(const ForwardArgs& a, cudaStream_t st);

// Tensor-core attention kernel (forward_tc.cu); `flag` is the validation result, the
// first word of the forward workspace.
size_t forward_tc_workspace(const Shape& s);
cudaError_t launch_forward_tc(const ForwardArgs& a, const int32_t* flag, cudaStream_t st);

// The attention kernel of the keep-or-drop and PISA modes at head dim 64
// (forward_pair.cu): kb16, vs16 [BH, Mp, d] and hb16 [BH, d, d] are the bf16 statistics
// (PISA only).
cudaError_t launch_forward_pair(const ForwardArgs& a, const int32_t* flag, const void* kb16,
                                const void* vs16, const void* hb16, int Mp, cudaStream_t st);

}  // namespace bsa
