/*
 * fmoe_gdn.h -- C ABI of libfmoe.so, part 2: the Gated DeltaNet state update of the
 * linear-attention layers at decode time, as a hand-written CUDA kernel for sm_100a.
 *
 * "What is Flash-MoE" (a2a-mcp.org), section 4 (Accelerate BLAS for the Gated DeltaNet
 * layers), and the "Flash-MoE" wiki summary (jeongsk), key technique 4: 45 of the 60
 * layers of Qwen3.5-397B-A17B are linear attention; each keeps a 128 x 128 state matrix
 * per head, 64 heads, and updates it for every token with a scaling, a matrix-vector
 * product and a rank-1 update (sscal, sgemv and sger, single precision, in the pages'
 * CPU code).  Read as the gated delta rule, per head:
 *   S <- alpha S                    (the gate decays the memory)
 *   u  = S k                        (what the memory returns for key k)
 *   S <- S + beta (v - u) k^T       (the delta rule's correction toward v)
 *   o  = S q                        (the read-out for query q)
 * i.e. S' = alpha S (I - beta k k^T) + beta v k^T and o = S' q.  The projections that
 * make q, k, v, alpha and beta, their normalisation and the output gate of the layer are
 * not part of this call.
 *
 * Conventions as in fmoe.h: device pointers owned by the caller, stream-ordered and
 * asynchronous, arguments checked on the host before anything is enqueued, no call
 * allocates, aborts or exits.
 */
#ifndef FMOE_GDN_H
#define FMOE_GDN_H

#include "fmoe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* flags of fmoe_gdn_step: the launch enqueued on `stream` just before this call does not
 * write `state` (in a model it is the projection that makes q, k, v of this layer); the
 * kernel may then read the state while that launch is still finishing, and waits for it
 * (dependent launch) only before it reads q, k, v, alpha and beta.  Without the flag the
 * kernel reads nothing before its predecessor is complete. */
#define FMOE_GDN_STATE_EARLY 1u

/* One decode step of n independent heads (a batch of B sequences with H heads each is
 * n = B * H heads), all in one launch:
 *   state: fp32 [n][dv][dk], row-major (row i of head h at (h * dv + i) * dk), read and
 *          written in place; 16-byte aligned.
 *   q, k:  fp32 [n][dk], 16-byte aligned.   v: fp32 [n][dv].   alpha, beta: fp32 [n].
 *   o:     fp32 [n][dv] (may be v itself; no other overlap).  v, alpha, beta, o 4-byte aligned.
 * Arithmetic: fp32 as the pages' BLAS calls, one fused pass per state row (fma, partial
 * sums per lane then a tree over the row); it agrees with the fp64 definition above to a
 * bound that grows with dk (the tests state it).
 * Requirements: n >= 0 (n = 0 enqueues nothing), dk in {128, 256, 384, 512}, dv >= 1,
 * n * dv < 2^31; flags 0 or FMOE_GDN_STATE_EARLY.
 * Errors: FMOE_ERR_INVALID_ARG (NULL pointer with n > 0, n < 0, dv < 1, unknown flags),
 * FMOE_ERR_UNSUPPORTED (dk, too many rows), FMOE_ERR_ALIGNMENT, FMOE_ERR_CUDA (launch). */
fmoe_status fmoe_gdn_step(float* state, const float* q, const float* k, const float* v, const float* alpha,
                          const float* beta, float* o, int n, int dk, int dv, unsigned flags, fmoe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_GDN_H */
