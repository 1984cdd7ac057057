/*
 * frnnt test hooks -- building blocks of frnnt_fwd_bwd exposed so the test
 * suite can check each kernel family on its own.  Not needed to use the
 * library; same ownership rules as frnnt.h (device pointers, caller-owned,
 * stream-ordered, nothing allocated).
 */
#ifndef FRNNT_TESTING_H
#define FRNNT_TESTING_H

#include "frnnt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The tensor-core (tcgen05 + TMA) bf16 GEMM used for the joint's
 * contractions and the projections:  D[M,N] = A[M,K] * B[K,N], fp32
 * accumulation.  A is K-major ([M][lda], a_mn = 0) or MN-major ([K][lda],
 * a_mn = 1); B is K-major ([N][ldb], b_mn = 0) or MN-major ([K][ldb]).
 * epi: 0 = store fp32 to out[M][ldo]; 1 = store bf16; 2 = fp32 atomic add
 * into out (k_splits >= 1 K slices); 3 = out (bf16, holding h on entry)
 * becomes D * (1 - h*h).  Requires lda, ldb multiples of 8, N a multiple of
 * 32, 16-byte aligned pointers.  variant: -1 automatic, 0 one CTA per 128-row
 * tile, 1 CTA pairs sharing 256-row tiles (cta_group::2); 2 / 3 as 0 / 1 with
 * 256-wide N tiles whatever N (a ragged last tile).  Returns FRNNT_OK or an
 * FRNNT_ERR_* code. */
FRNNT_API int frnnt_test_gemm_bf16(int M, int N, int K, const void* A, int a_mn, long long lda,
                                   const void* B, int b_mn, long long ldb, int epi, int k_splits,
                                   void* out, long long ldo, int variant, int32_t* status, void* stream);

/* Selects the fused joint kernel's variant for the frnnt_fwd_bwd calls that
 * follow (process-wide, not thread-safe; set it between calls): -1 automatic
 * (the default), 0 one CTA per 128-cell tile, 1 CTA pairs (a 2-CTA cluster,
 * each CTA its own cell tile and half of every W_o tile, M = 256 cta_group::2
 * MMAs).  Out-of-range values clamp to the nearest.  Returns the previous
 * setting.  Results of the two variants agree up to the order of fp32 atomic
 * additions. */
FRNNT_API int frnnt_test_joint_variant(int variant);

/* Failure-detection test setting: each of the next n tensor-core GEMM launches
 * (frnnt_test_gemm_bf16, or the GEMMs inside frnnt_fwd_bwd*) has every CTA
 * skip the load of its first K block, and the arrival that would announce it,
 * so the MMA issuer's bounded wait on that stage runs out (about 2 s).  The
 * kernel then stops every role, frees its tensor memory and ORs
 * FRNNT_STATUS_TIMEOUT into the call's status word (when one is given); the
 * context stays usable and later launches run normally.  That GEMM's output is
 * left incomplete.  n <= 0 clears the setting.  Process-wide, not thread-safe
 * (set it between calls).  Returns the previous count. */
FRNNT_API int frnnt_test_lose_gemm_loads(int n);

/* The K-slice count the tensor-core GEMM takes for a split-K launch (host
 * only, no GPU needed): mn output tiles on `workers` persistent CTAs (or CTA
 * pairs), kblocks K blocks of 64.  It minimises rounds x (K blocks per unit +
 * a fixed 64-block unit cost), the fewest slices on a tie; always in
 * [1, max(kblocks, 1)]. */
FRNNT_API int frnnt_test_auto_splits(int mn, int workers, int kblocks);

#ifdef __cplusplus
}
#endif
#endif /* FRNNT_TESTING_H */
