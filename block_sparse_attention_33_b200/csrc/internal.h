// Internal launch interface shared by the spattn translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace spattn {

enum { ROUTING_CENTROID = 0, ROUTING_PAMA = 1 };

// Device error code of the probe correction (after DEV_OK, DEV_BAD_INDEX and
// DEV_TIMEOUT): normal equations that are not positive definite.
enum : int { DEV_NUMERIC = 3 };

// Problem description derived from a plan (all sizes in elements).
struct Problem {
  int B, H, N, d, b, nb, n_last, kcap;
  int BH;
  float tau;
  int kmin, kmax;
  int residual;
  int use_tc;           // attention on the tcgen05 kernel (else warp MMA)
  int routing;          // ROUTING_CENTROID or ROUTING_PAMA
  int threshold;        // selection: 0 Top-p (tau = mass), 1 per-block p >= tau
  int inline_sel;       // 1: the attention kernel selects (no routing launch)
  int test_stall;       // failure-path test: CTA 0 of the attention waits on a phase
                        // that never completes, so its bounded wait runs out
  const int32_t* perm;  // device, NULL if none
};

// Device buffers of one workspace (pointers into it).
struct Work {
  __nv_bfloat16 *qp, *kp, *vp;  // permuted copies (NULL without perm)
  float *qbar, *kbar, *vbar;    // fp32 means [BH, nb, d]
  __nv_bfloat16 *kbar16, *vbar16;  // bf16 means for the residual tiles
  int32_t* counts;   // [BH*nb] kept count per query block
  int32_t* lists;    // [BH*nb*kcap] kept blocks, ascending, padded rows
  int32_t* row_ptr;  // [BH*nb + 1]
  int32_t* col_idx;  // [BH*nb*kcap]
  int32_t* order;    // [BH*nb] work order for the attention kernel
  int32_t* ctrl;     // control block (CTRL_WORDS int32)
};

cudaError_t launch_pool(const Problem& p, const void* Q, const void* K, const void* V,
                        const Work& w, cudaStream_t s);
// need_csr: also build the compact CSR in w.row_ptr / w.col_idx (the
// tcgen05 attention reads the padded per-row lists directly, so the compact
// copy is made only for callers and paths that need it).
// Q: the original queries (PAMA reads tokens through p.perm).
cudaError_t launch_route(const Problem& p, const Work& w, const void* Q, int32_t* row_ptr_out,
                         int32_t* col_idx_out, bool need_csr, cudaStream_t s);
cudaError_t launch_attend(const Problem& p, const void* Q, const void* K, const void* V,
                          const int32_t* row_ptr, const int32_t* col_idx, void* O,
                          const Work& w, cudaStream_t s);

// Exact softmax attention of gathered query rows (Qg: [BH, q_alloc, d] bf16,
// q_alloc a multiple of 128) over all N keys of K and V, fp32 output rows
// [BH, q_rows, d]; the tcgen05 attention kernel in its dense mode.
cudaError_t launch_dense_rows_tc(const Problem& p, const void* Qg, int q_alloc, int q_rows,
                                 const void* K, const void* V, float* out, float* part, float* lse,
                                 int32_t* ctrl, cudaStream_t s);
// key ranges a dense tile item may be cut into (part / lse buffers of the
// dense rows hold this many copies)
constexpr int DENSE_MAX_SPLITS = 8;

// O <- O + O W + c for every row of every head, on the tensor cores: Wt is
// bf16 [BH, d, d] holding W transposed (row n = column n of W), c fp32 [BH, d].
cudaError_t launch_probe_apply_tc(const Problem& p, void* O, const void* Wt, const float* c,
                                  int32_t* ctrl, cudaStream_t s);

// Probe-fitted residual correction (SparsePR page, section 2B) of the routed
// output O in place; scratch of probe_scratch_bytes(p, M) bytes.
size_t probe_scratch_bytes(const Problem& p, int M);
cudaError_t launch_probe_correct(const Problem& p, const void* Q, const void* K, const void* V,
                                 void* O, const int32_t* probes, int M, float lam, int r,
                                 void* scratch, int32_t* ctrl, cudaStream_t s);

// Raise kernel `fn`'s dynamic shared-memory limit on the current device to at
// least `bytes`; the attribute call is made only when a launch needs more
// than was granted before (thread-safe).
cudaError_t ensure_dyn_smem(const void* fn, size_t bytes);

}  // namespace spattn
