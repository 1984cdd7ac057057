// CUDA-core (SIMT, fp32 arithmetic) kernels: the FRNNT_F32 path, and a
// second independent GPU path for bf16 inputs (FRNNT_PATH_SIMT).
//
// The joint is evaluated exactly as defined -- h = tanh(F[t] + G[u]),
// z = h W_o^T + b_o per lattice cell ("Transformer Transducer", abstract:
// the two encoders' activations combined by a feed-forward layer for every
// (frame, label history) pair) -- over contiguous chunks of the padded cell
// index c = (b*T + t)*(U+1) + u, with plain tiled GEMMs for the
// contractions.
#include "frnnt_common.cuh"
#include "frnnt_internal.h"

namespace frnnt {

// ------------------------------------------------------------------ GEMM
namespace {
constexpr int GBM = 64, GBN = 64, GBK = 16;

template <typename TA, typename TB, bool TRA, bool TRB>
__global__ void __launch_bounds__(256) gemm_simt_kernel(int M, int N, int K, const TA* __restrict__ A, int lda,
                                                        const TB* __restrict__ Bm, int ldb, float* __restrict__ C,
                                                        int ldc, int accumulate) {
  __shared__ float As[GBK][GBM + 4];
  __shared__ float Bs[GBK][GBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const long long m0 = (long long)blockIdx.y * GBM, n0 = (long long)blockIdx.x * GBN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += GBK) {
    for (int i = tid; i < GBM * GBK; i += 256) {
      int mm, kk;
      if (TRA) { mm = i % GBM; kk = i / GBM; } else { kk = i % GBK; mm = i / GBK; }
      long long m = m0 + mm;
      int k = k0 + kk;
      float v = 0.f;
      if (m < M && k < K) v = to_f32(TRA ? A[(size_t)k * lda + m] : A[(size_t)m * lda + k]);
      As[kk][mm] = v;
    }
    for (int i = tid; i < GBN * GBK; i += 256) {
      int nn, kk;
      if (TRB) { kk = i % GBK; nn = i / GBK; } else { nn = i % GBN; kk = i / GBN; }
      long long n = n0 + nn;
      int k = k0 + kk;
      float v = 0.f;
      if (n < N && k < K) v = to_f32(TRB ? Bm[(size_t)n * ldb + k] : Bm[(size_t)k * ldb + n]);
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    long long m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      long long n = n0 + tx + 16 * j;
      if (n >= N) continue;
      float* p = C + (size_t)m * ldc + n;
      *p = accumulate ? *p + acc[i][j] : acc[i][j];
    }
  }
}

template <typename TA, typename TB>
void gemm_dispatch_t(int M, int N, int K, const void* A, int lda, bool tA, const void* B, int ldb, bool tB, float* C,
                     int ldc, bool acc, cudaStream_t st) {
  dim3 grid((N + GBN - 1) / GBN, (M + GBM - 1) / GBM);
  const TA* a = (const TA*)A;
  const TB* b = (const TB*)B;
  if (!tA && !tB) gemm_simt_kernel<TA, TB, false, false><<<grid, 256, 0, st>>>(M, N, K, a, lda, b, ldb, C, ldc, acc);
  else if (!tA && tB) gemm_simt_kernel<TA, TB, false, true><<<grid, 256, 0, st>>>(M, N, K, a, lda, b, ldb, C, ldc, acc);
  else if (tA && !tB) gemm_simt_kernel<TA, TB, true, false><<<grid, 256, 0, st>>>(M, N, K, a, lda, b, ldb, C, ldc, acc);
  else gemm_simt_kernel<TA, TB, true, true><<<grid, 256, 0, st>>>(M, N, K, a, lda, b, ldb, C, ldc, acc);
  note_launch();
}
}  // namespace

void launch_gemm_simt(int M, int N, int K, const void* A, int lda, bool a_bf16, bool transA, const void* B, int ldb,
                      bool b_bf16, bool transB, float* C, int ldc, bool accumulate, cudaStream_t st) {
  if (M <= 0 || N <= 0) return;
  using bf = __nv_bfloat16;
  if (a_bf16 && b_bf16) gemm_dispatch_t<bf, bf>(M, N, K, A, lda, transA, B, ldb, transB, C, ldc, accumulate, st);
  if (a_bf16 && !b_bf16) gemm_dispatch_t<bf, float>(M, N, K, A, lda, transA, B, ldb, transB, C, ldc, accumulate, st);
  if (!a_bf16 && b_bf16) gemm_dispatch_t<float, bf>(M, N, K, A, lda, transA, B, ldb, transB, C, ldc, accumulate, st);
  if (!a_bf16 && !b_bf16)
    gemm_dispatch_t<float, float>(M, N, K, A, lda, transA, B, ldb, transB, C, ldc, accumulate, st);
}

// ------------------------------------------------------------------ hidden
__global__ void hidden_simt_kernel(int T, int U, int H, const float* __restrict__ F, const float* __restrict__ G,
                                   const int32_t* __restrict__ T_len, const int32_t* __restrict__ U_len,
                                   long long c0, long long C, float* __restrict__ h) {
  const long long r = blockIdx.x;            // chunk row (one cell)
  if (r >= C) return;
  const long long c = c0 + r;
  const int Up1 = U + 1;
  const int u = (int)(c % Up1);
  const long long bt = c / Up1;
  const int b = (int)(bt / T), t = (int)(bt % T);
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const bool valid = t < l.Tb && u <= l.Ub;
  const float* Fr = F + (size_t)bt * H;
  const float* Gr = G + ((size_t)b * Up1 + u) * H;
  float* hr = h + (size_t)r * H;
  for (int j = threadIdx.x; j < H; j += blockDim.x) hr[j] = valid ? tanhf(Fr[j] + Gr[j]) : 0.f;
}

void launch_hidden_simt(const Shape& s, const float* F, const float* G, const int32_t* T_len, const int32_t* U_len,
                        long long c0, long long C, float* h, cudaStream_t st) {
  if (C <= 0) return;
  hidden_simt_kernel<<<(unsigned)C, 128, 0, st>>>(s.T, s.U, s.H, F, G, T_len, U_len, c0, C, h);
  note_launch();
}

// ------------------------------------------------------------------ reductions
__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
  for (int o = 16; o > 0; o >>= 1) {
    float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = lane < nw ? red[lane] : (is_max ? -INFINITY : 0.f);
  for (int o = 16; o > 0; o >>= 1) {
    float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  return v;
}

template <typename TW>
__global__ void lse_simt_kernel(int T, int U, int V, int blank, float* __restrict__ z, const TW* __restrict__ b_o,
                                const int32_t* __restrict__ labels, const int32_t* __restrict__ T_len,
                                const int32_t* __restrict__ U_len, long long c0, long long C, Lattice L) {
  __shared__ float red[32];
  const long long r = blockIdx.x;
  const long long c = c0 + r;
  const int Up1 = U + 1;
  const int u = (int)(c % Up1);
  const long long bt = c / Up1;
  const int b = (int)(bt / T), t = (int)(bt % T);
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  if (!(t < l.Tb && u <= l.Ub)) return;      // block-uniform
  float* zr = z + (size_t)r * V;
  float m = -INFINITY;
  for (int k = threadIdx.x; k < V; k += blockDim.x) {
    float v = zr[k] + to_f32(b_o[k]);
    zr[k] = v;
    m = fmaxf(m, v);
  }
  m = block_reduce(m, true, red);
  float sum = 0.f;
  for (int k = threadIdx.x; k < V; k += blockDim.x) sum += __expf(zr[k] - m);
  sum = block_reduce(sum, false, red);
  if (threadIdx.x == 0) {
    float lse = m + logf(sum);
    L.lse[c] = lse;
    L.blank_lp[c] = zr[blank] - lse;
    L.label_lp[c] = u < l.Ub ? zr[label_of(labels, b, u, U, V)] - lse : -INFINITY;
  }
}

void launch_lse_simt(const Shape& s, float* z, const void* b_o, const int32_t* labels, const int32_t* T_len,
                     const int32_t* U_len, long long c0, long long C, const Lattice& L, cudaStream_t st) {
  if (C <= 0) return;
  if (s.bf16)
    lse_simt_kernel<__nv_bfloat16><<<(unsigned)C, 128, 0, st>>>(s.T, s.U, s.V, s.blank, z,
                                                                (const __nv_bfloat16*)b_o, labels, T_len, U_len,
                                                                c0, C, L);
  else
    lse_simt_kernel<float><<<(unsigned)C, 128, 0, st>>>(s.T, s.U, s.V, s.blank, z, (const float*)b_o, labels,
                                                        T_len, U_len, c0, C, L);
  note_launch();
}

// ------------------------------------------------------------------ dz
// Posterior of the two edges leaving cell (t,u):
//   bpost = exp(alpha(t,u) + blank_lp(t,u) + beta'(t+1,u) - logP)   (beta'(T_len,U_len) = 0)
//   lpost = exp(alpha(t,u) + label_lp(t,u) + beta(t,u+1) - logP)    (u < U_len)
// dz_k = w_b (occ softmax_k - bpost [k = blank] - lpost [k = y_u]), occ = bpost + lpost.
constexpr int DZ_ROWS = 16;

template <typename TW>
__global__ void dz_simt_kernel(int T, int U, int V, int blank, float* __restrict__ z, int add_bias,
                               const TW* __restrict__ b_o, const int32_t* __restrict__ labels,
                               const int32_t* __restrict__ T_len, const int32_t* __restrict__ U_len,
                               const float* __restrict__ grad_loss, long long c0, long long C, Lattice L,
                               float* __restrict__ db_o) {
  extern __shared__ float dbs[];             // [V] partial column sums of this block
  for (int k = threadIdx.x; k < V; k += blockDim.x) dbs[k] = 0.f;
  __syncthreads();
  const int Up1 = U + 1;
  for (int rr = 0; rr < DZ_ROWS; ++rr) {
    const long long r = (long long)blockIdx.x * DZ_ROWS + rr;
    if (r >= C) break;
    const long long c = c0 + r;
    const int u = (int)(c % Up1);
    const long long bt = c / Up1;
    const int b = (int)(bt / T), t = (int)(bt % T);
    const Lengths l = lengths_of(T_len, U_len, b, T, U);
    float* zr = z + (size_t)r * V;
    if (!(t < l.Tb && u <= l.Ub)) {
      for (int k = threadIdx.x; k < V; k += blockDim.x) zr[k] = 0.f;
      continue;
    }
    float bpost, lpost;
    edge_posteriors(L, c, (size_t)b * T * Up1, t + 1 < l.Tb ? (long long)(c + Up1) : -1LL,
                    u < l.Ub ? (long long)(c + 1) : -1LL, t == l.Tb - 1 && u == l.Ub, bpost, lpost);
    const float occ = bpost + lpost;
    const float w = grad_loss ? grad_loss[b] : 1.f;
    const float lse = L.lse[c];
    const int y = u < l.Ub ? label_of(labels, b, u, U, V) : -1;
    for (int k = threadIdx.x; k < V; k += blockDim.x) {
      float v = zr[k] + (add_bias ? to_f32(b_o[k]) : 0.f);
      float d = occ * __expf(v - lse);
      if (k == blank) d -= bpost;
      if (k == y) d -= lpost;
      d *= w;
      zr[k] = d;
      dbs[k] += d;
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < V; k += blockDim.x) atomicAdd(db_o + k, dbs[k]);
}

void launch_dz_simt(const Shape& s, float* z, bool add_bias, const void* b_o, const int32_t* labels,
                    const int32_t* T_len, const int32_t* U_len, const float* grad_loss, long long c0, long long C,
                    const Lattice& L, float* db_o_acc, cudaStream_t st) {
  if (C <= 0) return;
  unsigned blocks = (unsigned)((C + DZ_ROWS - 1) / DZ_ROWS);
  size_t smem = (size_t)s.V * sizeof(float);
  if (s.bf16)
    dz_simt_kernel<__nv_bfloat16><<<blocks, 256, smem, st>>>(s.T, s.U, s.V, s.blank, z, add_bias,
                                                             (const __nv_bfloat16*)b_o, labels, T_len, U_len,
                                                             grad_loss, c0, C, L, db_o_acc);
  else
    dz_simt_kernel<float><<<blocks, 256, smem, st>>>(s.T, s.U, s.V, s.blank, z, add_bias, (const float*)b_o, labels,
                                                     T_len, U_len, grad_loss, c0, C, L, db_o_acc);
  note_launch();
}

// ------------------------------------------------------------------ dtanh + segmented sums
// Chunks are whole (b,t) rows of U+1 cells, so dF rows are complete in a chunk.
__global__ void dF_simt_kernel(int U, int H, const float* __restrict__ dh, const float* __restrict__ h,
                               long long row0, long long nrows, float* __restrict__ dF) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nrows * H) return;
  const long long r = i / H;
  const int j = (int)(i % H);
  const int Up1 = U + 1;
  float s = 0.f;
  for (int u = 0; u < Up1; ++u) {
    size_t o = ((size_t)r * Up1 + u) * H + j;
    float hv = h[o];
    s += dh[o] * (1.f - hv * hv);
  }
  dF[(size_t)(row0 + r) * H + j] = s;
}

__global__ void dG_simt_kernel(int T, int U, int H, const float* __restrict__ dh, const float* __restrict__ h,
                               long long row0, long long nrows, float* __restrict__ dG) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int Up1 = U + 1;
  if (i >= (long long)Up1 * H) return;
  const int u = (int)(i / H), j = (int)(i % H);
  int cur_b = -1;
  float s = 0.f;
  for (long long r = 0; r < nrows; ++r) {
    const int b = (int)((row0 + r) / T);
    if (b != cur_b) {
      if (cur_b >= 0) atomicAdd(dG + ((size_t)cur_b * Up1 + u) * H + j, s);
      cur_b = b;
      s = 0.f;
    }
    size_t o = ((size_t)r * Up1 + u) * H + j;
    float hv = h[o];
    s += dh[o] * (1.f - hv * hv);
  }
  if (cur_b >= 0) atomicAdd(dG + ((size_t)cur_b * Up1 + u) * H + j, s);
}

void launch_dtanh_reduce_simt(const Shape& s, const float* dh, const float* h, long long c0, long long C, float* dF,
                              float* dG, cudaStream_t st) {
  if (C <= 0) return;
  const long long row0 = c0 / s.Up1, nrows = C / s.Up1;
  long long n1 = nrows * s.H;
  dF_simt_kernel<<<(unsigned)((n1 + 255) / 256), 256, 0, st>>>(s.U, s.H, dh, h, row0, nrows, dF);
  note_launch();
  long long n2 = (long long)s.Up1 * s.H;
  dG_simt_kernel<<<(unsigned)((n2 + 255) / 256), 256, 0, st>>>(s.T, s.U, s.H, dh, h, row0, nrows, dG);
  note_launch();
}

// ------------------------------------------------------------------ convert
__global__ void convert_kernel(const float* __restrict__ in, void* __restrict__ out, long long n, int to_bf16) {
  chain_wait();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    if (to_bf16) ((__nv_bfloat16*)out)[i] = __float2bfloat16_rn(in[i]);
    else ((float*)out)[i] = in[i];
  }
}

void launch_convert(const float* in, void* out, long long n, bool to_bf16, cudaStream_t st) {
  if (n <= 0) return;
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  launch_k(convert_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 1, in, out, n, to_bf16);
  note_launch();
}

void launch_convert_bf16(const float* in, void* out, long long n, cudaStream_t st) {
  launch_convert(in, out, n, true, st);
}

}  // namespace frnnt
