/*
 * spattn -- routed block-sparse attention with proxy residual, for NVIDIA
 * B200 (sm_100a).  C ABI.
 *
 * What the library computes (one attention call; pages: PARK "Accurate
 * Block Retrieval for Sparse Attention in Video Diffusion Transformers",
 * sections 3.1-3.2 and D.2; Sol-Attn abstract; DFSAttn abstract):
 *
 *   Q, K, V: bf16 [B, H, N, d] (row-major, d contiguous).  With a token
 *   permutation perm, tokens are first gathered, Xp[n] = X[perm[n]].
 *   Tokens are cut into nb = ceil(N / b) blocks; block j holds n_j tokens
 *   (b, except a possibly partial last block).  Query blocks use the same
 *   partition.
 *
 *   1. block means Qbar_i, Kbar_j, Vbar_j in fp32;
 *   2. proxy logits s_ij = Qbar_i . Kbar_j / sqrt(d) + ln n_j and
 *      p_ij = softmax_j(s_ij) (PARK 3.2 block importance; the ln n_j term
 *      makes s_ij the Jensen lower bound of PARK D.2);
 *   3. per query block i, blocks in descending p (ties: lower j) and the
 *      shortest prefix whose cumulative mass reaches tau is kept, budget
 *      clamped to [kmin, min(kmax, nb)]; tau >= 1 keeps every block
 *      (PARK 3.2 "Top-p"; Sol-Attn dynamic budgets);
 *   4. each query token q of block i runs one softmax over the exact tokens
 *      of its kept blocks; with residual != 0 every dropped block j adds one
 *      pseudo-key with logit q . Kbar_j / sqrt(d) + ln n_j and value Vbar_j
 *      (Sol-Attn abstract: skipped blocks approximated from the router's scores);
 *   5. the output is scattered back, O[perm[n]] = Op[n], bf16.
 *
 * Conventions for every call:
 *   - Pointers named *_host are host memory; every other data pointer is
 *     device memory of the current CUDA device.  The caller owns all of
 *     them; the library keeps no pointer past the call that received it.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Device
 *     work is enqueued on it and the call returns without waiting;
 *     argument errors are reported synchronously before anything is
 *     enqueued.
 *   - Every call returns a spattn_status_t; spattn_last_error() gives a
 *     human-readable message for the calling thread's last failure.  No
 *     C++ exception crosses this boundary.
 *   - CUDA graphs: spattn_pool, spattn_route, spattn_attend, spattn_forward,
 *     spattn_means and spattn_probe_correct enqueue kernels and async copies
 *     only, so they can be captured once each has run eagerly with the same
 *     plan (the first call may raise a kernel's shared-memory limit and, for
 *     spattn_probe_correct, does so for its kernels).  spattn_plan (device
 *     allocation with a permutation), spattn_check (synchronises),
 *     spattn_forward_host (creates streams and events) and the first
 *     spattn_route_static call on a device are not capturable.
 *   - Supported: d in {64, 128}; b in {64, 128}; 1 <= N; nb <= 2048;
 *     1 <= kmin <= kmax (kmax > nb is clamped to nb); tau finite;
 *     B*H <= 65535; B*H*nb*min(kmax, nb) <= 2^31 - 1 (int32 CSR offsets).
 */
#ifndef SPATTN_H_
#define SPATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPATTN_OK = 0,
  SPATTN_ERR_INVALID_ARG = 1,  /* bad shape, knob, pointer or permutation */
  SPATTN_ERR_UNSUPPORTED = 2,  /* valid but outside the supported range  */
  SPATTN_ERR_WORKSPACE = 3,    /* workspace missing or too small          */
  SPATTN_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed       */
  SPATTN_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up      */
  SPATTN_ERR_DEVICE = 6        /* a kernel flagged bad data (e.g. a CSR
                                  block index out of range); see
                                  spattn_check                             */
} spattn_status_t;

typedef struct spattn_plan_s* spattn_plan_t;

/* Create a plan for one problem shape and set of routing knobs.
 *   B, H, N, d, b       shapes (see above);
 *   tau, kmin, kmax     Top-p threshold and budget clamp;
 *   residual            0: dropped blocks are skipped; 1: pseudo-keys;
 *   perm_host           NULL, or N int32 forming a bijection of [0, N):
 *                       perm[new] = old.  The plan copies it to device
 *                       memory it owns (this needs a current CUDA device);
 *   workspace_bytes     out: bytes of device workspace the route/attend/
 *                       forward calls need (256-byte aligned base).
 * (Failure-path test: with SPATTN_TEST_FAIL_ALLOC=1 in the environment, the
 * device allocation of the permutation reports out-of-memory without being
 * attempted, and the call returns SPATTN_ERR_CUDA with no plan.)
 * Validation happens before any CUDA call.  The plan is immutable and may
 * be shared by threads; one workspace must not be used by two calls that
 * overlap on the device. */
spattn_status_t spattn_plan(spattn_plan_t* out, int B, int H, int N, int d, int b,
                            float tau, int kmin, int kmax, int residual,
                            const int32_t* perm_host, size_t* workspace_bytes);

/* Block-importance estimate that drives the Top-p selection. */
enum {
  SPATTN_ROUTING_CENTROID = 0, /* p_i = softmax_j(Qbar_i . Kbar_j / sqrt(d) + ln n_j):
                                  block-mean query and key centroids (PARK page
                                  3.2 block importance from centroids)           */
  SPATTN_ROUTING_PAMA = 1      /* p_i = mean over the tokens q of block i of
                                  softmax_j(q . Kbar_j / sqrt(d) + ln n_j): each
                                  query keeps its own normalisation (PARK page
                                  5.1, per-query attention-mass aggregation);
                                  costs 2 * n_i * nb * d FMAs per query block
                                  (two passes), on fp32 lanes                   */
};

/* Selection flag, OR'ed into the routing argument of spattn_plan_ex.  With
 * it, tau is read as a per-block probability threshold theta: block j of
 * query block i is kept iff p_ij >= theta (theta <= 0 keeps every block),
 * and the budget is clamped to [kmin, min(kmax, nb)] in the Top-p order
 * (p descending, ties to the lower j) when a clamp binds.  This is the
 * on-the-fly block thresholding of the Sol-Attn abstract (thelatestinai
 * page), which gives no rule for the threshold: a fixed threshold on p is
 * the reading taken here.  Dropped blocks take the residual pseudo-keys as
 * before. */
enum { SPATTN_SELECT_THRESHOLD = 16 };

/* Selection flag, OR'ed into the routing argument of spattn_plan_ex (with
 * the centroid estimate, optionally with SPATTN_SELECT_THRESHOLD): the
 * attention kernel selects the blocks itself, inside the attention pass
 * (Sol-Attn abstract, thelatestinai page: critical blocks are chosen by
 * comparing proxy scores with a threshold during the online softmax, without
 * materialising the proxy map).  Per work item the kernel scores its query
 * block against every key block from the fp32 means, forms the block softmax
 * and cuts the row (threshold theta = tau, or Top-p mass tau, with the same
 * clamp), in on-chip memory only, with the same arithmetic as the routing
 * kernel, so it keeps exactly the blocks spattn_route would list.  With it:
 *   spattn_forward  is spattn_pool + the attention: no routing launch, no
 *                   kept lists, no CSR;
 *   spattn_attend   with NULL row_ptr / col_idx selects from the means the
 *                   last spattn_pool or spattn_route left in the workspace
 *                   (a caller CSR is used as given);
 *   spattn_route    still writes the CSR of the same selection, for callers
 *                   that want to see it.
 * The budget of every query block is found per work item, so the work runs
 * in plain (batch, head, block) order rather than longest-first. */
enum { SPATTN_SELECT_INLINE = 32 };

/* spattn_plan with a choice of routing estimate (one of the values above,
 * optionally | SPATTN_SELECT_THRESHOLD and, with the centroid estimate,
 * | SPATTN_SELECT_INLINE; anything else is SPATTN_ERR_INVALID_ARG).  spattn_plan is
 * spattn_plan_ex(..., SPATTN_ROUTING_CENTROID, ...).  spattn_route_static
 * always uses the centroid estimate and the Top-p selection. */
spattn_status_t spattn_plan_ex(spattn_plan_t* out, int B, int H, int N, int d, int b,
                               float tau, int kmin, int kmax, int residual,
                               const int32_t* perm_host, int routing, size_t* workspace_bytes);

/* Release a plan (and its device copy of the permutation). NULL is a no-op. */
spattn_status_t spattn_plan_destroy(spattn_plan_t plan);

/* Number of query/key blocks nb and the capacity (B*H*nb*min(kmax, nb)) a
 * caller-provided col_idx buffer must have. */
spattn_status_t spattn_plan_info(spattn_plan_t plan, int* nb, int64_t* col_capacity);

/* Gather (if the plan has a permutation) and pool.  Writes the permuted
 * copies of Q, K, V (read by the attention as whole tiles) and the fp32 block
 * means Qbar, Kbar, Vbar (with bf16 copies of Kbar, Vbar for the residual
 * tiles) into the workspace.  Q, K, V: bf16 [B, H, N, d] device. */
spattn_status_t spattn_pool(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                            void* workspace, void* stream);

/* spattn_pool, then proxy scoring, Top-p selection and the CSR
 * of kept blocks.  spattn_pool and spattn_route clear the workspace's
 * device error word first.
 *   row_ptr  NULL or int32 [B*H*nb + 1], rows ordered (batch, head, block i);
 *   col_idx  NULL or int32 [col capacity], kept block indices j in [0, nb),
 *            ascending within a row.
 * The kept lists are always also left in the workspace (padded per row)
 * for a following attend. */
spattn_status_t spattn_route(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                             void* workspace, int32_t* row_ptr, int32_t* col_idx,
                             void* stream);

/* Routed attention (+ residual pseudo-keys) and the scatter
 * of the output, using the permuted copies and block means that the last
 * spattn_pool / spattn_route left in this workspace for the same inputs.
 * Routing reuse across calls (SVOO and PARK reuse sparse masks across
 * diffusion steps): after one spattn_route, a spattn_pool on new inputs
 * followed by spattn_attend with NULL row_ptr/col_idx attends the new
 * inputs with the kept lists of that earlier route (the residual uses the
 * new inputs' means).
 *   row_ptr, col_idx  NULL to use the kept lists the last spattn_route left
 *                     in the workspace, or a caller CSR in the layout above
 *                     (device).  The caller guarantees row_ptr[0] = 0, a
 *                     non-decreasing row_ptr, at most nb entries per row,
 *                     and a col_idx that holds every entry row_ptr
 *                     points at: the library cannot see the size of a device
 *                     buffer and reads col_idx[row_ptr[r] .. row_ptr[r+1]).
 *                     With b = 128 a block listed twice is attended twice;
 *                     with b = 64 two query blocks share their key tiles
 *                     and a block listed twice counts once.  Block
 *                     indices outside [0, nb) are skipped and flagged
 *                     (SPATTN_ERR_DEVICE from spattn_check).  With a
 *                     caller CSR the call first clears the workspace's
 *                     device error word (the workspace may never have
 *                     been routed); without a permutation and with
 *                     residual = 0 it then needs nothing else from an
 *                     earlier call.
 *   O                 bf16 [B, H, N, d] device, written in the original
 *                     token order. */
spattn_status_t spattn_attend(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                              const int32_t* row_ptr, const int32_t* col_idx, void* O,
                              void* workspace, void* stream);

/* The whole path: spattn_route (kept lists in the workspace only) +
 * spattn_attend. */
spattn_status_t spattn_forward(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                               void* O, void* workspace, void* stream);

/* Device staging bytes spattn_forward_host needs for chunks of chunk_heads
 * (batch, head) pairs (chunk_heads >= 1; values above B*H count as B*H, and
 * so does any chunk too large for the workspace to hold a chunk's scratch
 * beside the plan's error word, which only happens on tiny problems): two
 * slots of the chunk's Q, K, V and O. */
spattn_status_t spattn_host_staging_bytes(spattn_plan_t plan, int chunk_heads, size_t* bytes);

/* spattn_forward on HOST-resident tensors, with the transfers overlapped.
 * The pages say nothing on this; it exists because heads are independent
 * through the whole path, so the copy of one chunk of heads in, the path on
 * the previous chunk and the copy of the chunk before it out can run at
 * once instead of one after the other.
 *   Q_host, K_host, V_host  bf16 [B, H, N, d] host memory (pinned memory
 *                           lets the copies run asynchronously; pageable
 *                           memory works but the copies then block);
 *   O_host                  bf16 [B, H, N, d] host memory, written;
 *   workspace               as for spattn_forward (workspace_bytes);
 *   staging                 device, spattn_host_staging_bytes(plan,
 *                           chunk_heads) bytes, 256-byte aligned;
 *   chunk_heads             (batch, head) pairs per chunk, >= 1.
 * Chunk g (heads g*c .. g*c+c-1 in (batch, head) order) is copied into one of
 * two staging slots on a copy stream, run through pool, route and attend on
 * `stream`, and copied out on a second copy stream; slots are reused two
 * chunks later.  The output equals spattn_forward's bit for bit.  The call
 * returns after enqueueing; synchronise `stream` before reading O_host or
 * reusing the input buffers.  spattn_check reports the first device error
 * of any chunk.  The host buffers must stay valid until then; on an error
 * status, synchronise the device before reusing any of the buffers. */
spattn_status_t spattn_forward_host(spattn_plan_t plan, const void* Q_host, const void* K_host,
                                    const void* V_host, void* O_host, void* workspace,
                                    void* staging, int chunk_heads, void* stream);

/* Device scratch bytes spattn_probe_correct needs for M probe rows per
 * (batch, head) pair. */
spattn_status_t spattn_probe_scratch_bytes(spattn_plan_t plan, int M, size_t* bytes);

/* Probe-fitted residual correction of a routed output, in place (SparsePR
 * page, section 2B: a few query rows are evaluated exactly, the residual
 * R = O_dense - O_sparse of those rows is fitted as an affine function
 * b + x B of the sparse output by ridge regression, the fitted correction is
 * restricted to the span of the r leading right singular vectors of R, and
 * it is added to every row; probe rows take their exact output).  Per
 * (batch, head) pair:
 *   Q, K, V   bf16 [B, H, N, d] device, original token order (the inputs of
 *             the spattn_forward that produced O);
 *   O         bf16 [B, H, N, d] device: in, the routed output; out, the
 *             corrected output;
 *   probes    int32 [B, H, M] device token indices in [0, N) (the page
 *             stratifies them across query groups; the caller chooses them).
 *             An index outside [0, N) is skipped and flagged (spattn_check:
 *             SPATTN_ERR_DEVICE);
 *   lam       ridge penalty on B (>= 0; the bias b is not penalised);
 *   r         0 <= r <= d: rank of the residual subspace (0: no correction
 *             off the probes; d: the whole output space);
 *   workspace the plan's workspace (its device error word only);
 *   scratch   device, spattn_probe_scratch_bytes(plan, M) bytes, 256-byte
 *             aligned.
 * The exact probe rows run on the tensor cores, as the attention does (bf16
 * operands, fp32 accumulation), with an fp32 output.  The fit is fp32: one
 * Gram pass over the probe rows [1, x, R] gives the (d+1) x (d+1) normal
 * equations (inverted by Gauss-Jordan elimination) and R^T R, whose r leading
 * eigenvectors come from block subspace iteration with a Rayleigh-Ritz step
 * (r + 16 <= d / 2; cyclic Jacobi on the whole matrix otherwise).  The pass
 * O += O (B P) + b P runs on the tensor cores with B P in bf16 (the
 * correction is a small fraction of the output) and fp32 accumulation.  Normal
 * equations that are not positive definite (lam = 0 with fewer than d + 1
 * independent probe rows, for instance), or a fit or subspace that is not
 * finite, leave that head uncorrected and are flagged (spattn_check:
 * SPATTN_ERR_DEVICE).  B*H <= 65535. */
spattn_status_t spattn_probe_correct(spattn_plan_t plan, const void* Q, const void* K,
                                     const void* V, void* O, const int32_t* probes, int M,
                                     float lam, int r, void* workspace, void* scratch,
                                     void* stream);

/* Copy the fp32 block means [B, H, nb, d] left in the workspace by the last
 * pool/route into caller device buffers (any may be NULL). */
spattn_status_t spattn_means(spattn_plan_t plan, const void* workspace, float* Qbar,
                             float* Kbar, float* Vbar, void* stream);

/* Synchronise `stream` and report the device error word of this workspace:
 * SPATTN_OK, SPATTN_ERR_DEVICE or SPATTN_ERR_TIMEOUT.  Clears the word.
 * (To exercise the timeout path without a fault: with the environment
 * variable SPATTN_TEST_WAIT_TIMEOUT=1 set when a plan is made, the first CTA
 * of that plan's attention waits on a phase nothing completes, gives up
 * after about two seconds, and this call then reports SPATTN_ERR_TIMEOUT.) */
spattn_status_t spattn_check(spattn_plan_t plan, void* workspace, void* stream);

/* Host helper (no CUDA): perm[new] = old ordering the tokens of a T x Hs x W
 * latent grid (row-major token order n = (t*Hs + h)*W + w) along a 3D
 * Hilbert curve (DFSAttn abstract: Hilbert curve-based token reordering).
 * The curve is J. Skilling's ("Programming the Hilbert curve", AIP Conf.
 * Proc. 707, 2004) on the smallest power-of-two cube covering the grid,
 * axes (t, h, w); tokens are stably sorted by curve index.  perm_host must
 * hold T*Hs*W int32.  A grid side above 2^21 is SPATTN_ERR_UNSUPPORTED (the
 * curve index of three such axes would not fit 64 bits). */
spattn_status_t spattn_hilbert_perm(int T, int Hs, int W, int32_t* perm_host);

/* Routing without any device allocation (pooling of Q and K, scoring,
 * selection and CSR; no permuted copies).
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc: code whose device memory belongs to another
 * allocator that forbids side allocations, plug-ins that are handed only
 * their inputs and outputs, and loops that must not pay cudaMalloc's implicit
 * device synchronisation.  It computes the same CSR as spattn_route for the
 * same shape and knobs (same kernels, bit-identical result), without a plan
 * or workspace:
 *   B, H, N, d, b, tau, kmin, kmax   as for spattn_plan;
 *   perm     NULL, or a DEVICE array of N int32 (perm[new] = old), 4-byte
 *            aligned, which the caller guarantees to be a bijection (it is not
 *            checked on the host; an entry outside [0, N) is skipped by the
 *            pooling, never read through, and the CSR is then unspecified);
 *   Q, K     bf16 [B, H, N, d] device, 16-byte aligned (V is not needed);
 *   row_ptr  int32 [B*H*nb + 1] device, col_idx int32 [B*H*nb*min(kmax, nb)]
 *            device, both 4-byte aligned: the CSR, as written by spattn_route.
 * Scratch lives in one file-scope device array of
 * SPATTN_ROUTE_STATIC_SCRATCH_BYTES, held by every GPU that loads the library
 * until the process exits.  A problem needs
 *     256 + 2*up(R*d*4) + 2*up(R*4) + up(R*min(kmax, nb)*4)
 * bytes of it, with R = B*H*nb and up() rounding up to a multiple of 256 (a
 * control block, the fp32 means of Q and K, per-row budgets and work order,
 * padded kept lists); a problem that needs more is rejected with
 * SPATTN_ERR_UNSUPPORTED before any pointer is looked at or anything runs.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it; make that
 * first call before any stream capture, and do not use this entry point
 * across a cudaDeviceReset (the kept address would be stale).  Every call
 * shares the one array: calls that overlap on the GPU (other streams or host
 * threads) race and must be serialised by the caller.  Device-side errors
 * are not reported by this path (there is no workspace to hold them and no
 * check call for it).  No cudaMalloc, cudaFree or allocating library
 * routine is called. */
#define SPATTN_ROUTE_STATIC_SCRATCH_BYTES (32u << 20)
spattn_status_t spattn_route_static(int B, int H, int N, int d, int b, float tau, int kmin,
                                    int kmax, const int32_t* perm, const void* Q, const void* K,
                                    int32_t* row_ptr, int32_t* col_idx, void* stream);

/* Message for the calling thread's last non-OK status ("" if none). */
const char* spattn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SPATTN_H_ */
