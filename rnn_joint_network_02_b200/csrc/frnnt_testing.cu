// Test hooks of include/frnnt_testing.h.
#include "frnnt_internal.h"
#include "frnnt_testing.h"

extern "C" FRNNT_API int frnnt_test_gemm_bf16(int M, int N, int K, const void* A, int a_mn, long long lda,
                                              const void* B, int b_mn, long long ldb, int epi, int k_splits,
                                              void* out, long long ldo, int variant, int32_t* status,
                                              void* stream) {
  if (!A || !B || !out) return FRNNT_ERR_NULL;
  if (epi < 0 || epi > 3) return FRNNT_ERR_UNSUPPORTED;
  frnnt::GemmTcArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.A = A;
  g.a_mn = a_mn != 0;
  g.lda = lda;
  g.B = B;
  g.b_mn = b_mn != 0;
  g.ldb = ldb;
  g.epi = epi;
  g.k_splits = k_splits;
  g.out_f32 = (epi == 0 || epi == 2) ? (float*)out : nullptr;
  g.out_bf16 = (epi == 1 || epi == 3) ? out : nullptr;
  g.ldo = ldo;
  g.status = status;
  g.variant = variant < -1 || variant > 3 ? -1 : variant;
  cudaGetLastError();
  return frnnt::gemm_tc(g, (cudaStream_t)stream);
}

extern "C" FRNNT_API int frnnt_test_joint_variant(int variant) { return frnnt::set_joint_variant(variant); }

extern "C" FRNNT_API int frnnt_test_lose_gemm_loads(int n) { return frnnt::lose_gemm_loads(n); }

extern "C" FRNNT_API int frnnt_test_auto_splits(int mn, int workers, int kblocks) {
  return frnnt::auto_splits(mn, workers, kblocks);
}
