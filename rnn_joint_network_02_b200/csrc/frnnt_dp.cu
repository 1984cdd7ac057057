// Validation of lengths / labels and the transducer forward-backward over the
// (T_len, U_len+1) lattice.
//
// The lattice recursion is the transducer's ("Sequence Transduction with
// Recurrent Neural Networks", abstract: the loss sums over every alignment):
//   alpha(t,u) = lae(alpha(t-1,u) + blank_lp(t-1,u), alpha(t,u-1) + label_lp(t,u-1))
//   beta(t,u)  = lae(beta(t+1,u)  + blank_lp(t,u),   beta(t,u+1)  + label_lp(t,u))
// with alpha(0,0) = 0, beta(T-1,U) = blank_lp(T-1,U) and log P = beta(0,0).
//
// Schedule: an anti-diagonal wavefront.  Cells with the same d = t + u depend
// only on diagonal d-1 (alpha) or d+1 (beta), so one thread owns one label
// position u and walks the diagonals; the value it needs from its neighbour
// u-1 (alpha) or u+1 (beta) is the neighbour's result on the previous
// diagonal.  One block per (utterance, direction): alpha and beta run
// concurrently.  How the neighbour's value travels depends on the kernel:
//  * dp2_kernel (marginal loss) advances two diagonals per dependent step and
//    exchanges every neighbour value through a parity-double-buffered
//    shared-memory row (no shuffles, no warp-edge special cases);
//  * dp_viterbi_kernel (maximum approximation) passes it by a warp shuffle
//    inside a warp and by shared memory across warp boundaries;
//  * dp_band_warp_kernel (pruned band, one warp per utterance and direction)
//    scans the band with shuffles;
//  * tdt_dp_kernel (token-and-duration lattice) uses shared memory only.
#include "frnnt_common.cuh"
#include "frnnt_internal.h"

namespace frnnt {

__global__ void validate_kernel(int B, int T, int U, int V, int blank, const int32_t* __restrict__ labels,
                                const int32_t* __restrict__ T_len, const int32_t* __restrict__ U_len,
                                int32_t* __restrict__ status) {
  chain_wait();
  int bits = validate_bits(B, T, U, V, blank, labels, T_len, U_len, threadIdx.x, blockDim.x);
  bits = __reduce_or_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0 && bits) atomicOr(status, bits);
}

// Pruned lattice: the bands of every utterance with valid lengths must start
// at 0, stay within [0, U_len], advance by 0 .. S-1 per frame and reach U_len
// in the last frame (then an alignment inside the band exists).
__global__ void validate_bounds_kernel(int B, int T, int U, int S, const int32_t* __restrict__ bounds,
                                       const int32_t* __restrict__ T_len, const int32_t* __restrict__ U_len,
                                       int32_t* __restrict__ status) {
  chain_wait();
  int bad = 0;
  const long long n = (long long)B * T;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int b = (int)(i / T), t = (int)(i % T);
    const int tl = T_len[b], ul = U_len[b];
    if (tl < 1 || tl > T || ul < 0 || ul > U) continue;   // length already flagged
    if (t >= tl) continue;                                // padding frame
    const int s = bounds[i];
    if (s < 0 || s > ul) bad = 1;
    if (t == 0 && s != 0) bad = 1;
    if (t + 1 < tl) {
      const int sn = bounds[i + 1];
      if (sn < s || sn > s + S - 1) bad = 1;
    } else if (s + S - 1 < ul) {
      bad = 1;
    }
  }
  bad = __reduce_or_sync(0xffffffffu, bad);
  if ((threadIdx.x & 31) == 0 && bad) atomicOr(status, FRNNT_STATUS_BOUNDS);
}

void launch_validate_bounds(const Shape& s, const int32_t* bounds, const int32_t* T_len, const int32_t* U_len,
                            int32_t* status, cudaStream_t st) {
  const long long n = (long long)s.B * s.T;
  const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
  launch_k(validate_bounds_kernel, dim3(blocks), dim3(256), 0, st, 1, s.B, s.T, s.U, s.S, bounds, T_len, U_len, status);
  note_launch();
}

void launch_validate(const Shape& s, const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                     const int32_t* bounds, int32_t* status, cudaStream_t st) {
  launch_k(validate_kernel, dim3(1), dim3(256), 0, st, 1, s.B, s.T, s.U, s.V, s.blank, labels, T_len, U_len, status);
  note_launch();
  if (s.S > 0) {
    const long long n = (long long)s.B * s.T;
    const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
    launch_k(validate_bounds_kernel, dim3(blocks), dim3(256), 0, st, 1, s.B, s.T, s.U, s.S, bounds, T_len, U_len, status);
    note_launch();
  }
}

// Operands of step `step` for thread u: alpha needs blank_lp(t-1,u) and
// label_lp(t,u-1); beta needs blank_lp(t,u) and label_lp(t,u) (t = d - u).
// They do not depend on the recursion, so they are fetched kPrefetch steps
// ahead into a register ring to hide the global-memory latency.
constexpr int kPrefetch = 8;

__device__ __forceinline__ void dp_operands(bool is_beta, int step, int ndiag, int u, int Tb, int Ub, int Up1,
                                            size_t base, const float* __restrict__ blank_lp,
                                            const float* __restrict__ label_lp, float& ob, float& ol) {
  ob = 0.f;
  ol = 0.f;
  if (step >= ndiag) return;
  const int d = is_beta ? (ndiag - 1 - step) : step;
  const int t = d - u;
  if (u > Ub || t < 0 || t >= Tb) return;
  const size_t c = base + (size_t)t * Up1 + u;
  if (!is_beta) {
    if (t > 0) ob = __ldg(blank_lp + c - Up1);
    if (u > 0) ol = __ldg(label_lp + c - 1);
  } else {
    ob = __ldg(blank_lp + c);
    if (u < Ub) ol = __ldg(label_lp + c);
  }
}

// Two diagonals per step.  A cell on diagonal d+2 is reached from diagonal d
// by three two-edge paths whose weights use only the log-probabilities:
//   alpha(t,u) = lae(alpha(t-2,u)   + b(t-2,u) + b(t-1,u),
//                    alpha(t-1,u-1) + lae(b(t-1,u-1) + l(t,u-1), l(t-1,u-1) + b(t-1,u)),
//                    alpha(t,u-2)   + l(t,u-2) + l(t,u-1))
// (b = blank_lp, l = label_lp, -inf outside the lattice), and the middle
// diagonal d+1 takes the usual one-edge step from d as well.  Both depend on
// diagonal d only, so the dependent chain is one diagonal pair long instead
// of two diagonals.  Beta mirrors it:
//   beta(t,u)  = lae(beta(t+2,u)   + b(t,u) + b(t+1,u),
//                    beta(t+1,u+1) + lae(b(t,u) + l(t+1,u), l(t,u) + b(t,u+1)),
//                    beta(t,u+2)   + l(t,u) + l(t,u+1)).
// A thread owns label position u; the values of u-1, u-2 (alpha) or u+1, u+2
// (beta) on the previous diagonal pair come through a parity-double-buffered
// shared array with one entry per thread (one barrier per step, no shuffles).
// The six log-probabilities of a step are fetched kPrefetch2 steps ahead.
constexpr int kPrefetch2 = kDp2Prefetch;

struct DpOps {
  float bA, bB, bC, lA, lB, lC;
};

// alpha, cell (t,u) on diagonal d+2 (t = d + 2 - u):
//   bA = b(t-2,u), bB = b(t-1,u), bC = b(t-1,u-1), lA = l(t,u-1), lB = l(t-1,u-1), lC = l(t,u-2)
// beta, cell (t,u) on diagonal d-2:
//   bA = b(t,u), bB = b(t+1,u), bC = b(t,u+1), lA = l(t+1,u), lB = l(t,u), lC = l(t,u+1)
__device__ __forceinline__ float lp_at(const float* __restrict__ a, size_t base, int Up1, int t, int u, int Tb,
                                       int umax) {
  return (t >= 0 && t < Tb && u >= 0 && u <= umax) ? __ldg(a + base + (size_t)t * Up1 + u) : -INFINITY;
}

__device__ __forceinline__ DpOps dp2_operands(bool is_beta, int step, int nsteps, int u, int Tb, int Ub, int Up1,
                                              int last, size_t base, const float* __restrict__ blank_lp,
                                              const float* __restrict__ label_lp) {
  DpOps o{-INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
  if (step >= nsteps || u > Ub) return o;
  if (!is_beta) {
    const int t = 2 * step + 2 - u;           // cell on the far diagonal of this step
    o.bA = lp_at(blank_lp, base, Up1, t - 2, u, Tb, Ub);
    o.bB = lp_at(blank_lp, base, Up1, t - 1, u, Tb, Ub);
    o.bC = lp_at(blank_lp, base, Up1, t - 1, u - 1, Tb, Ub);
    o.lA = lp_at(label_lp, base, Up1, t, u - 1, Tb, Ub - 1);
    o.lB = lp_at(label_lp, base, Up1, t - 1, u - 1, Tb, Ub - 1);
    o.lC = lp_at(label_lp, base, Up1, t, u - 2, Tb, Ub - 1);
  } else {
    const int t = last - 2 * step - 2 - u;    // cell on the far diagonal of this step
    o.bA = lp_at(blank_lp, base, Up1, t, u, Tb, Ub);
    o.bB = lp_at(blank_lp, base, Up1, t + 1, u, Tb, Ub);
    o.bC = lp_at(blank_lp, base, Up1, t, u + 1, Tb, Ub);
    o.lA = lp_at(label_lp, base, Up1, t + 1, u, Tb, Ub - 1);
    o.lB = lp_at(label_lp, base, Up1, t, u, Tb, Ub - 1);
    o.lC = lp_at(label_lp, base, Up1, t, u + 1, Tb, Ub - 1);
  }
  return o;
}

// The five weights of a step (below) from its six log-probabilities.
__device__ __forceinline__ void dp2_step_weights(bool is_beta, int step, int nsteps, int last, int u, int Tb, int Ub,
                                                 const DpOps& o, float (&wv)[5]) {
  const bool live = step < nsteps && u <= Ub;
  if (!is_beta) {
    const int t = 2 * step + 2 - u;
    const bool mid = live && t - 1 >= 0 && t - 1 < Tb;
    const bool far = live && 2 * step + 2 <= last && t >= 0 && t < Tb;
    wv[0] = mid ? o.bA : -INFINITY;
    wv[1] = mid ? o.lB : -INFINITY;
    wv[2] = far ? o.bA + o.bB : -INFINITY;
    wv[3] = far ? log_add_exp(o.bC + o.lA, o.lB + o.bB) : -INFINITY;
    wv[4] = far ? o.lC + o.lA : -INFINITY;
  } else {
    const int t = last - 2 * step - 2 - u;
    const bool mid = live && t + 1 >= 0 && t + 1 < Tb;
    const bool far = live && last - 2 * step - 2 >= 0 && t >= 0 && t < Tb;
    wv[0] = mid ? o.bB : -INFINITY;
    wv[1] = mid ? o.lA : -INFINITY;
    wv[2] = far ? o.bA + o.bB : -INFINITY;
    wv[3] = far ? log_add_exp(o.bA + o.lA, o.lB + o.bC) : -INFINITY;
    wv[4] = far ? o.lB + o.lC : -INFINITY;
  }
}

// The step's weights, precomputed for every (utterance, direction, step, label
// position) by a parallel kernel, so that the serial wavefront loads five
// numbers per step with no index arithmetic or bounds checks on them:
//   alpha, far cell (t,u), t = 2 step + 2 - u, middle cell (t-1,u):
//     M1 = b(t-2,u), M2 = l(t-1,u-1);  W1 = b(t-2,u) + b(t-1,u),
//     W2 = lae(b(t-1,u-1) + l(t,u-1), l(t-1,u-1) + b(t-1,u)),  W3 = l(t,u-2) + l(t,u-1)
//   beta, far cell (t,u), t = last - 2 step - 2 - u, middle cell (t+1,u):
//     M1 = b(t+1,u), M2 = l(t+1,u);  W1 = b(t,u) + b(t+1,u),
//     W2 = lae(b(t,u) + l(t+1,u), l(t,u) + b(t,u+1)),  W3 = l(t,u) + l(t,u+1)
// so that middle = lae(cur + M1, n1 + M2) and far = lae(lae(cur + W1, n1 + W2), n2 + W3)
// (cur, n1, n2: the previous far diagonal at u and at u -/+ 1, 2), with all
// weights -inf for a cell outside the lattice, whose value then is -inf too.
// Layout [b][direction][step][5][UP] (UP = the DP's block size), with
// kPrefetch2 extra steps so that the prefetch never needs a bound.
__global__ void dp2_weights_kernel(int B, int T, int U, int NS, int UP, const float* __restrict__ blank_lp,
                                   const float* __restrict__ label_lp, const int32_t* __restrict__ T_len,
                                   const int32_t* __restrict__ U_len, float* __restrict__ w) {
  chain_wait();
  const long long n = (long long)B * 2 * NS * UP;
  const int Up1 = U + 1;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int u = (int)(i % UP);
    long long r = i / UP;
    const int step = (int)(r % NS);
    r /= NS;
    const bool is_beta = (r & 1) != 0;
    const int b = (int)(r >> 1);
    const Lengths l = lengths_of(T_len, U_len, b, T, U);
    const int Tb = l.Tb, Ub = l.Ub;
    const int last = Tb - 1 + Ub;
    const int nsteps = (last + 1) / 2;
    const size_t base = (size_t)b * T * Up1;
    const DpOps o = dp2_operands(is_beta, step, nsteps, u, Tb, Ub, Up1, last, base, blank_lp, label_lp);
    float wv[5];
    dp2_step_weights(is_beta, step, nsteps, last, u, Tb, Ub, o, wv);
    float* dst = w + ((size_t)(((long long)b * 2 + (is_beta ? 1 : 0)) * NS + step) * 5) * UP + u;
#pragma unroll
    for (int k = 0; k < 5; ++k) dst[k * UP] = wv[k];
  }
}

// PRE: the step weights come from dp2_weights_kernel (wts); otherwise each
// thread forms its own from the six log-probabilities of the step, fetched
// kPrefetch2 steps ahead (no weight array: the tiled mode's memory budget).
template <bool PRE>
__global__ void dp2_kernel(int T, int U, int NS, const float* __restrict__ blank_lp,
                           const float* __restrict__ label_lp, const float* __restrict__ wts,
                           float* __restrict__ alpha, float* __restrict__ beta, const int32_t* __restrict__ T_len,
                           const int32_t* __restrict__ U_len, float* __restrict__ loss) {
  chain_wait();
  __shared__ float xa[2][1024];     // [parity][thread]: each thread's value on the last far diagonal
  const int b = blockIdx.x;
  const bool is_beta = blockIdx.y == 1;
  const int u = threadIdx.x;
  const int nth = blockDim.x;       // = the weights' UP
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const int Tb = l.Tb, Ub = l.Ub;
  const int Up1 = U + 1;
  const size_t base = (size_t)b * T * Up1;
  const int last = Tb - 1 + Ub;             // the last diagonal
  const int nsteps = (last + 1) / 2;        // steps of two diagonals after diagonal 0 (alpha) / `last` (beta)
  const bool in_u = u <= Ub;
  const float* wp = PRE ? wts + (size_t)((long long)b * 2 + (is_beta ? 1 : 0)) * NS * 5 * nth + u : nullptr;

  // the first diagonal: (0,0) for alpha, (Tb-1, Ub) for beta
  float cur = -INFINITY;
  if (!is_beta) {
    if (u == 0) {
      cur = 0.f;
      alpha[base] = 0.f;
    }
  } else if (u == Ub) {
    const size_t c = base + (size_t)(Tb - 1) * Up1 + Ub;
    cur = __ldg(blank_lp + c);
    beta[c] = cur;
    if (last == 0) loss[b] = -cur;
  }

  float q[kPrefetch2][5];
  DpOps qo[PRE ? 1 : kPrefetch2];
  if constexpr (PRE) {
#pragma unroll
    for (int i = 0; i < kPrefetch2; ++i)
#pragma unroll
      for (int k = 0; k < 5; ++k) q[i][k] = __ldg(wp + (size_t)(i * 5 + k) * nth);
  } else {
#pragma unroll
    for (int i = 0; i < kPrefetch2; ++i)
      qo[i] = dp2_operands(is_beta, i, nsteps, u, Tb, Ub, Up1, last, base, blank_lp, label_lp);
  }

  // parity 1 holds the first diagonal
  xa[1][u] = cur;
  __syncthreads();

  for (int step0 = 0; step0 < nsteps; step0 += kPrefetch2) {
#pragma unroll
    for (int i = 0; i < kPrefetch2; ++i) {
      const int step = step0 + i;
      if (step >= nsteps) break;    // uniform across the block
      float m1, m2, w1, w2, w3;
      if constexpr (PRE) {
        m1 = q[i][0]; m2 = q[i][1]; w1 = q[i][2]; w2 = q[i][3]; w3 = q[i][4];
        // (NS covers nsteps + kPrefetch2 steps: no bound on the prefetch)
#pragma unroll
        for (int k = 0; k < 5; ++k) q[i][k] = __ldg(wp + (size_t)((step + kPrefetch2) * 5 + k) * nth);
      } else {
        float wv[5];
        dp2_step_weights(is_beta, step, nsteps, last, u, Tb, Ub, qo[i], wv);
        m1 = wv[0]; m2 = wv[1]; w1 = wv[2]; w2 = wv[3]; w3 = wv[4];
        qo[i] = dp2_operands(is_beta, step + kPrefetch2, nsteps, u, Tb, Ub, Up1, last, base, blank_lp, label_lp);
      }
      const int par = (step + 1) & 1;       // parity holding the previous pair's far values
      float n1, n2;                          // neighbours at distance 1 and 2 on the previous far diagonal
      if (!is_beta) {
        n1 = u >= 1 ? xa[par][u - 1] : -INFINITY;
        n2 = u >= 2 ? xa[par][u - 2] : -INFINITY;
      } else {
        n1 = u + 1 < nth ? xa[par][u + 1] : -INFINITY;
        n2 = u + 2 < nth ? xa[par][u + 2] : -INFINITY;
      }
      const float v1 = log_add_exp(cur + m1, n1 + m2);
      const float v2 = log_add_exp(log_add_exp(cur + w1, n1 + w2), n2 + w3);
      if (in_u) {
        if (!is_beta) {
          const int t1 = 2 * step + 1 - u, t2 = t1 + 1;
          if (t1 >= 0 && t1 < Tb) alpha[base + (size_t)t1 * Up1 + u] = v1;
          if (2 * step + 2 <= last && t2 >= 0 && t2 < Tb) alpha[base + (size_t)t2 * Up1 + u] = v2;
        } else {
          const int d2 = last - 2 * step - 2;
          const int t2 = d2 - u, t1 = t2 + 1;
          if (t1 >= 0 && t1 < Tb) beta[base + (size_t)t1 * Up1 + u] = v1;
          if (d2 >= 0 && t2 >= 0 && t2 < Tb) {
            beta[base + (size_t)t2 * Up1 + u] = v2;
            if (t2 == 0 && u == 0) loss[b] = -v2;
          }
          if (d2 < 0 && t1 == 0 && u == 0) loss[b] = -v1;
        }
      }
      // the far diagonal of this step becomes the previous one (the middle one
      // when the far one is past the lattice's end)
      const bool far_exists = is_beta ? (last - 2 * step - 2 >= 0) : (2 * step + 2 <= last);
      cur = far_exists ? v2 : v1;
      xa[step & 1][u] = cur;
      __syncthreads();
    }
  }
}

// Maximum approximation: the alpha wavefront with max in place of log-add-exp
// (same schedule as dp_kernel's alpha block), recording for every cell
// whether its best predecessor is the blank edge from (t-1, u) (ties go to
// the blank edge); then one thread walks the best alignment back from
// (T_len-1, U_len), marking the edge by which it leaves each cell on it.
// The decisions go to a shared-memory bit array (one bit per padded cell of
// the utterance) when `smem_bits`, so the walk reads no global memory;
// otherwise to bit 2 of the path bytes.
__global__ void dp_viterbi_kernel(int T, int U, const float* __restrict__ blank_lp,
                                  const float* __restrict__ label_lp, float* __restrict__ alpha,
                                  uint8_t* __restrict__ path, const int32_t* __restrict__ T_len,
                                  const int32_t* __restrict__ U_len, float* __restrict__ loss, int smem_bits) {
  chain_wait();
  __shared__ float xs[2][32];
  extern __shared__ uint32_t dec_bits[];   // smem_bits: ceil(T (U+1) / 32) words
  const int b = blockIdx.x;
  const int u = threadIdx.x;
  const int lane = u & 31, warp = u >> 5;
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const int Tb = l.Tb, Ub = l.Ub;
  const int Up1 = U + 1;
  const size_t base = (size_t)b * T * Up1;
  const int ndiag = Tb + Ub;
  if (smem_bits) {
    const int nwords = (T * Up1 + 31) / 32;
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) dec_bits[i] = 0u;
    __syncthreads();
  }

  float qb[kPrefetch], ql[kPrefetch];
#pragma unroll
  for (int i = 0; i < kPrefetch; ++i)
    dp_operands(false, i, ndiag, u, Tb, Ub, Up1, base, blank_lp, label_lp, qb[i], ql[i]);

  float cur = -INFINITY;
  for (int step0 = 0; step0 < ndiag; step0 += kPrefetch) {
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) {
      const int step = step0 + i;
      if (step >= ndiag) break;     // uniform across the block
      const float ob = qb[i], ol = ql[i];
      dp_operands(false, step + kPrefetch, ndiag, u, Tb, Ub, Up1, base, blank_lp, label_lp, qb[i], ql[i]);
      const int t = step - u;
      const bool active = (u <= Ub) && (t >= 0) && (t < Tb);
      float nb = __shfl_up_sync(0xffffffffu, cur, 1);
      if (lane == 0) nb = warp > 0 ? xs[(step + 1) & 1][warp - 1] : -INFINITY;
      float v = -INFINITY;
      if (active) {
        const size_t c = base + (size_t)t * Up1 + u;
        bool from_blank = false;
        if (t == 0 && u == 0) {
          v = 0.f;
        } else {
          const float fb = t > 0 ? cur + ob : -INFINITY;   // from (t-1, u)
          const float fl = u > 0 ? nb + ol : -INFINITY;    // from (t, u-1)
          from_blank = fb >= fl;
          v = from_blank ? fb : fl;
        }
        alpha[c] = v;
        if (smem_bits) {
          path[c] = 0;
          if (from_blank) {
            const int idx = t * Up1 + u;
            atomicOr(&dec_bits[idx >> 5], 1u << (idx & 31));
          }
        } else {
          path[c] = from_blank ? 4 : 0;
        }
      }
      cur = v;
      if (lane == 31) xs[step & 1][warp] = cur;
      __syncthreads();
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const size_t cl = base + (size_t)(Tb - 1) * Up1 + Ub;
    loss[b] = -(alpha[cl] + blank_lp[cl]);
    path[cl] |= 1;                  // the final blank
    int t = Tb - 1, uu = Ub;
    while (t > 0 || uu > 0) {       // t + uu falls by one per step
      const size_t c = base + (size_t)t * Up1 + uu;
      const int idx = t * Up1 + uu;
      const bool by_blank = smem_bits ? ((dec_bits[idx >> 5] >> (idx & 31)) & 1u) != 0 : (path[c] & 4) != 0;
      // the predecessor's edge bit (a plain store when the decisions are in
      // shared memory: the byte was zeroed by the wavefront)
      size_t pc;
      uint8_t bit;
      if (by_blank && t > 0) {
        --t;
        pc = c - Up1;
        bit = 1;
      } else if (uu > 0) {
        --uu;
        pc = c - 1;
        bit = 2;
      } else {
        --t;                        // not reached with finite log-probs
        pc = c - Up1;
        bit = 1;
      }
      if (smem_bits) path[pc] = bit;
      else path[pc] |= bit;
    }
  }
}

// Pruned lattice (layout [b][t][j], label position u = s[b,t] + j, j < S).
// One thread per (utterance, direction) walks the band row by row; the
// previous row (alpha) or next row (beta) is kept in shared memory.  A cell
// (t, u) is in the lattice when t < T_len, j < S and u <= U_len; its blank
// predecessor (t-1, u) sits at j' = u - s[b,t-1] of the previous row when
// 0 <= j' < S.  With `viterbi`, alpha takes the max (ties to the blank edge),
// the decision goes to bit 2 of the path byte, and the alpha thread then walks
// the best alignment back, marking the edge that leaves each cell on it.
__global__ void dp_band_kernel(int T, int U, int S, const int32_t* __restrict__ bounds,
                               const float* __restrict__ blank_lp, const float* __restrict__ label_lp,
                               float* __restrict__ alpha, float* __restrict__ beta, uint8_t* __restrict__ path,
                               const int32_t* __restrict__ T_len, const int32_t* __restrict__ U_len,
                               float* __restrict__ loss) {
  chain_wait();
  __shared__ float row[2][32];      // [direction][j] of the neighbouring row
  const int b = blockIdx.x;
  const int dir = threadIdx.x;      // 0 alpha, 1 beta
  const bool viterbi = path != nullptr;
  if (dir > 1 || (viterbi && dir == 1)) return;
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const int Tb = l.Tb, Ub = l.Ub;
  const size_t base = (size_t)b * T * S;
  const int32_t* sb = bounds + (size_t)b * T;
  float* prev = row[dir];
  if (dir == 0) {
    int sp = 0;
    for (int t = 0; t < Tb; ++t) {
      const int s = clampi(sb[t], 0, U);
      float left = -INFINITY;       // alpha(t, u-1) within this row
      float cur_row[32];
#pragma unroll 1
      for (int j = 0; j < S; ++j) {
        const int u = s + j;
        const size_t c = base + (size_t)t * S + j;
        float v = -INFINITY;
        bool from_blank = false;
        if (u <= Ub) {
          if (t == 0 && u == 0) {
            v = 0.f;
          } else {
            float fb = -INFINITY;
            const int jp = u - sp;
            if (t > 0 && jp >= 0 && jp < S) fb = prev[jp] + __ldg(blank_lp + base + (size_t)(t - 1) * S + jp);
            const float fl = j > 0 ? left + __ldg(label_lp + c - 1) : -INFINITY;
            if (viterbi) {
              from_blank = fb >= fl;
              v = from_blank ? fb : fl;
            } else {
              v = log_add_exp(fb, fl);
            }
          }
        }
        alpha[c] = v;
        if (viterbi) path[c] = from_blank ? 4 : 0;
        cur_row[j] = v;
        left = v;
      }
#pragma unroll 1
      for (int j = 0; j < S; ++j) prev[j] = cur_row[j];
      sp = s;
    }
    const int jl = Ub - clampi(sb[Tb - 1], 0, U);
    if (viterbi && jl >= 0 && jl < S) {   // (invalid bounds are flagged; nothing to walk then)
      size_t c = base + (size_t)(Tb - 1) * S + jl;
      loss[b] = -(alpha[c] + __ldg(blank_lp + c));
      path[c] |= 1;                 // the final blank
      int t = Tb - 1, u = Ub;
      while (t > 0 || u > 0) {      // t + u falls by one per step
        const int s = clampi(sb[t], 0, U);
        if ((path[c] & 4) && t > 0) {
          const int jp = u - clampi(sb[t - 1], 0, U);
          if (jp < 0 || jp >= S) break;   // not reached with valid bounds
          --t;
          c = base + (size_t)t * S + jp;
          path[c] |= 1;
        } else if (u > s) {
          --u;
          c -= 1;
          path[c] |= 2;
        } else {
          break;                    // not reached with valid bounds
        }
      }
    }
  } else {
    int sn = 0;
    for (int t = Tb - 1; t >= 0; --t) {
      const int s = clampi(sb[t], 0, U);
      float right = -INFINITY;      // beta(t, u+1) within this row
      float cur_row[32];
#pragma unroll 1
      for (int j = S - 1; j >= 0; --j) {
        const int u = s + j;
        const size_t c = base + (size_t)t * S + j;
        float v = -INFINITY;
        if (u <= Ub) {
          if (t == Tb - 1 && u == Ub) {
            v = __ldg(blank_lp + c);
          } else {
            float bb = -INFINITY;
            const int jn = u - sn;
            if (t + 1 < Tb && jn >= 0 && jn < S) bb = prev[jn] + __ldg(blank_lp + c);
            const float bl = (j + 1 < S && u + 1 <= Ub) ? right + __ldg(label_lp + c) : -INFINITY;
            v = log_add_exp(bb, bl);
          }
        }
        beta[c] = v;
        cur_row[j] = v;
        right = v;
      }
#pragma unroll 1
      for (int j = 0; j < S; ++j) prev[j] = cur_row[j];
      sn = s;
    }
    loss[b] = -beta[base];
  }
}

// The same pruned recursion with one warp per (utterance, direction) and lane
// j = band position (S <= 32): a frame's blank-edge terms come from the
// neighbouring frame by one shuffle (the band moves by bounds[t] - bounds[t-1],
// the same for every lane); the label-edge recurrence along the frame,
// x_j = lae(a_j, x_{j-1} + l_{j-1}), is an inclusive scan over lanes with the
// associative composition of the maps x -> lae(a, x + l):
//   (a1, l1) then (a2, l2)  =  (lae(a2, a1 + l2), l1 + l2)
// (max for the maximum approximation).  Beta runs the mirrored scan from the
// right.  The next frame's operands are fetched one frame ahead.  With
// `viterbi` the decision bits of each frame (a ballot) go to shared memory and
// lane 0 walks the best alignment back.
__device__ __forceinline__ float comb(bool viterbi, float a, float b) { return viterbi ? fmaxf(a, b) : log_add_exp(a, b); }

// SP: the band width rounded up to a power of two (4 .. 32): the scan's levels
// are unrolled (levels past S leave the band's lanes unchanged), and a lane
// that takes no part in a level keeps its value by a select, not a branch.
template <int SP>
__global__ void __launch_bounds__(32) dp_band_warp_kernel(int T, int U, int S, const int32_t* __restrict__ bounds,
                                                          const float* __restrict__ blank_lp,
                                                          const float* __restrict__ label_lp, float* __restrict__ alpha,
                                                          float* __restrict__ beta, uint8_t* __restrict__ path,
                                                          const int32_t* __restrict__ T_len,
                                                          const int32_t* __restrict__ U_len, float* __restrict__ loss) {
  chain_wait();
  // shared memory: the utterance's band starts (T ints), then (viterbi) one
  // ballot of decisions per frame (T words)
  extern __shared__ int32_t dsm[];
  int32_t* starts = dsm;
  uint32_t* dec = (uint32_t*)(dsm + T);
  const int b = blockIdx.x;
  const bool is_beta = blockIdx.y == 1;
  const bool viterbi = path != nullptr;
  const int lane = threadIdx.x;
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const int Tb = l.Tb, Ub = l.Ub;
  const size_t base = (size_t)b * T * S;
  for (int t = lane; t < Tb; t += 32) starts[t] = clampi(bounds[(size_t)b * T + t], 0, U);
  __syncwarp();
  auto start = [&](int t) { return starts[t]; };
  if (!is_beta) {
    // operands of frame t: blank_lp(t-1, u) at the previous frame's position and label_lp(t, u-1)
    auto fetch = [&](int t, float& ob, float& ol) {
      ob = -INFINITY;
      ol = -INFINITY;
      if (t >= Tb) return;
      const int s = start(t), u = s + lane;
      if (lane >= S || u > Ub) return;
      if (t > 0) {
        const int jp = u - start(t - 1);
        if (jp >= 0 && jp < S) ob = __ldg(blank_lp + base + (size_t)(t - 1) * S + jp);
      }
      if (lane > 0) ol = __ldg(label_lp + base + (size_t)t * S + lane - 1);
    };
    // operands fetched two frames ahead
    float ob, ol, ob1, ol1, ob2, ol2;
    fetch(0, ob, ol);
    fetch(1, ob1, ol1);
    float prev = -INFINITY;
    int sp = 0;
    for (int t = 0; t < Tb; ++t) {
      fetch(t + 2, ob2, ol2);
      const int s = start(t), u = s + lane;
      const bool valid = lane < S && u <= Ub;
      const int delta = s - sp;
      const int src = lane + delta < 32 ? lane + delta : 31;
      const float pv = __shfl_sync(0xffffffffu, prev, src);
      const float fb = (t > 0 && valid && lane + delta < S) ? pv + ob : -INFINITY;
      float a = (t == 0 && u == 0) ? 0.f : fb;
      float c = ol;
      float x = a;
      // inclusive scan over lanes (the band's S lanes need log2 S steps)
#pragma unroll
      for (int off = 1; off < SP; off <<= 1) {
        const float xa = __shfl_up_sync(0xffffffffu, x, off);
        const float xc = __shfl_up_sync(0xffffffffu, c, off);
        const bool in = lane >= off;
        const float xn = comb(viterbi, x, xa + c);
        c = in ? xc + c : c;
        x = in ? xn : x;
      }
      if (!valid) x = -INFINITY;
      if (lane < S) {
        alpha[base + (size_t)t * S + lane] = x;
        if (viterbi) path[base + (size_t)t * S + lane] = 0;
      }
      if (viterbi) {
        const float left = __shfl_up_sync(0xffffffffu, x, 1);
        const bool from_blank = valid && (lane == 0 || fb >= left + ol);
        const uint32_t bits = __ballot_sync(0xffffffffu, from_blank);
        if (lane == 0) dec[t] = bits;
      }
      prev = x;
      sp = s;
      ob = ob1;
      ol = ol1;
      ob1 = ob2;
      ol1 = ol2;
    }
    if (viterbi) {
      __syncwarp();
      if (lane == 0) {
        int t = Tb - 1;
        int j = Ub - start(t);
        if (j >= 0 && j < S) {
          size_t c = base + (size_t)t * S + j;
          loss[b] = -(alpha[c] + __ldg(blank_lp + c));
          path[c] = 1;              // the final blank
          while (t > 0 || start(t) + j > 0) {
            if (((dec[t] >> j) & 1u) && t > 0) {
              const int u = start(t) + j;
              const int jp = u - start(t - 1);
              if (jp < 0 || jp >= S) break;   // not reached with valid bounds
              --t;
              j = jp;
              c = base + (size_t)t * S + j;
              path[c] = 1;
            } else if (j > 0) {
              --j;
              c -= 1;
              path[c] = 2;
            } else {
              break;                // not reached with valid bounds
            }
          }
        }
      }
    }
  } else {
    // operands of frame t: blank_lp(t, u) and label_lp(t, u)
    auto fetch = [&](int t, float& ob, float& ol) {
      ob = -INFINITY;
      ol = -INFINITY;
      if (t < 0) return;
      const int u = start(t) + lane;
      if (lane >= S || u > Ub) return;
      ob = __ldg(blank_lp + base + (size_t)t * S + lane);
      if (lane + 1 < S && u < Ub) ol = __ldg(label_lp + base + (size_t)t * S + lane);
    };
    float ob, ol, ob1, ol1, ob2, ol2;
    fetch(Tb - 1, ob, ol);
    fetch(Tb - 2, ob1, ol1);
    float next = -INFINITY;
    int sn = 0;
    for (int t = Tb - 1; t >= 0; --t) {
      fetch(t - 2, ob2, ol2);
      const int s = start(t), u = s + lane;
      const bool valid = lane < S && u <= Ub;
      const int d2 = (t + 1 < Tb) ? sn - s : 0;
      const int src = lane - d2 >= 0 ? lane - d2 : 0;
      const float nv = __shfl_sync(0xffffffffu, next, src);
      float bb = (t + 1 < Tb && valid && lane - d2 >= 0) ? nv + ob : -INFINITY;
      if (t == Tb - 1 && u == Ub) bb = ob;   // the final blank
      float y = valid ? bb : -INFINITY;
      float c = ol;
      // inclusive scan from the right
#pragma unroll
      for (int off = 1; off < SP; off <<= 1) {
        const float ya = __shfl_down_sync(0xffffffffu, y, off);
        const float yc = __shfl_down_sync(0xffffffffu, c, off);
        const bool in = lane + off < 32;
        const float yn = comb(false, y, c + ya);
        c = in ? c + yc : c;
        y = in ? yn : y;
      }
      if (!valid) y = -INFINITY;
      if (lane < S) beta[base + (size_t)t * S + lane] = y;
      next = y;
      sn = s;
      ob = ob1;
      ol = ol1;
      ob1 = ob2;
      ol1 = ol2;
    }
    if (lane == 0) loss[b] = -beta[base];
  }
}

// ------------------------------------------------------------------ token-and-duration lattice
// "Efficient Sequence Transduction by Jointly Predicting Tokens and Durations"
// (abstract): every emission also draws a duration, the number of frames it
// covers.  From cell (t,u) a label with duration k goes to (t+k, u+1), a blank
// with duration k >= 1 to (t+k, u), each edge weighing
// token_lp + dur_lp(k); alignments end with a blank from (t, U_len) that lands
// exactly on frame T_len.
//
// Cells still form anti-diagonal wavefronts (an edge of duration k advances
// the diagonal by k or k+1), so one thread again owns one label position u:
//  * alpha pushes.  Once alpha(t,u) is known the thread adds its blank edges
//    into a shift register of its own future diagonals (fut[k] = diagonal
//    s+k) and hands its label edges, one per duration, to thread u+1 through
//    shared memory, which adds them to its own register one diagonal later.
//    Only the cell's own log-probs are read.
//  * beta pulls.  The thread keeps its own beta of the last DM+1 diagonals in
//    a shift register (hist[k] = diagonal s+k) and reads thread u+1's
//    register (through shared memory) for the label edges; (T_len, U_len) after the final blank is a
//    virtual cell with beta 0 on diagonal T_len + U_len.  It stores PB / PL
//    (the blank / label parts of beta) and, per duration, the log posterior
//    numerator without alpha and log P.
// DM = the largest duration (1..8): register arrays are indexed by compile-time k.
// Every thread exchanges through a parity-double-buffered shared array
// xa[parity][k][thread] (one barrier per step, no shuffles): dynamic shared
// memory of 2 (DM+2) blockDim floats.
// exp2 / log2 by the hardware approximations (ex2(-inf) = 0, lg2(0) = -inf)
constexpr float kLog2eDp = 1.4426950408889634f;
constexpr float kLn2Dp = 0.6931471805599453f;
__device__ __forceinline__ float ex2_dp(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_dp(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int DM>
struct TdtOps {
  float bl, ll;
  float dl[DM + 1];    // -inf for durations outside the set
};

template <int DM>
__device__ __forceinline__ void tdt_operands(TdtOps<DM>& o, bool live, int t, int u, int Tb, int Ub, int Up1,
                                             size_t base, long long plane, uint32_t dmask,
                                             const float* __restrict__ blank_lp, const float* __restrict__ label_lp,
                                             const float* __restrict__ dur_lp) {
  o.bl = -INFINITY;
  o.ll = -INFINITY;
#pragma unroll
  for (int k = 0; k <= DM; ++k) o.dl[k] = -INFINITY;
  if (!live || u > Ub || t < 0 || t >= Tb) return;
  const size_t c = base + (size_t)t * Up1 + u;
  o.bl = __ldg(blank_lp + c);
  if (u < Ub) o.ll = __ldg(label_lp + c);
  int i = 0;
#pragma unroll
  for (int k = 0; k <= DM; ++k)
    if ((dmask >> k) & 1u) {
      o.dl[k] = __ldg(dur_lp + (size_t)i * plane + c);
      ++i;
    }
}

constexpr int tdt_prefetch(int DM) { return DM <= 4 ? 4 : 2; }

// MAXT: the block size bound (256 and 512 let the registers hold every array without spilling).
template <int DM, int MAXT>
__global__ void __launch_bounds__(MAXT) tdt_dp_kernel(int T, int U, uint32_t dmask, long long plane,
                                                      const float* __restrict__ blank_lp,
                                                      const float* __restrict__ label_lp,
                                                      const float* __restrict__ dur_lp, float* __restrict__ alpha,
                                                      float* __restrict__ beta_b, float* __restrict__ beta_l,
                                                      float* __restrict__ q, const int32_t* __restrict__ T_len,
                                                      const int32_t* __restrict__ U_len, float* __restrict__ loss) {
  chain_wait();
  constexpr int P = tdt_prefetch(DM);
  extern __shared__ float xa[];           // [2][DM+2][blockDim]
  const int b = blockIdx.x;
  const bool is_beta = blockIdx.y == 1;
  const int u = threadIdx.x;
  const int nth = blockDim.x;
  auto X = [&](int par, int k, int i) -> float& { return xa[(par * (DM + 2) + k) * nth + i]; };
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const int Tb = l.Tb, Ub = l.Ub;
  const int Up1 = U + 1;
  const size_t base = (size_t)b * T * Up1;
  const int last = Tb - 1 + Ub;           // the last diagonal
  const int nsteps = last + 1;
  // diagonal of step i: i (alpha) or last - i (beta); the thread's cell on it has t = diagonal - u
  auto cell_t = [&](int i) { return (is_beta ? last - i : i) - u; };

  TdtOps<DM> ops[P];
#pragma unroll
  for (int i = 0; i < P; ++i)
    tdt_operands<DM>(ops[i], i < nsteps, cell_t(i), u, Tb, Ub, Up1, base, plane, dmask, blank_lp, label_lp, dur_lp);

  if (!is_beta) {
    float fut[DM + 1];    // incoming weight of this thread's cell on diagonal s + k
#pragma unroll
    for (int k = 0; k <= DM; ++k) fut[k] = -INFINITY;
#pragma unroll
    for (int k = 0; k < DM + 2; ++k) X(1, k, u) = -INFINITY;
    __syncthreads();
    for (int s0 = 0; s0 < nsteps; s0 += P) {
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const int s = s0 + i;
        if (s >= nsteps) break;           // uniform across the block
        const TdtOps<DM> o = ops[i];
        tdt_operands<DM>(ops[i], s + P < nsteps, cell_t(s + P), u, Tb, Ub, Up1, base, plane, dmask, blank_lp,
                         label_lp, dur_lp);
        // label edges of thread u-1 from diagonal s-1 with duration k land on diagonal s + k
#pragma unroll
        for (int k = 0; k <= DM; ++k) {
          if (!((dmask >> k) & 1u)) continue;
          const float nl = u > 0 ? X((s + 1) & 1, k, u - 1) : -INFINITY;
          fut[k] = log_add_exp(fut[k], nl);
        }
        const int t = s - u;
        const bool valid = u <= Ub && t >= 0 && t < Tb;
        const float v = valid ? ((t == 0 && u == 0) ? 0.f : fut[0]) : -INFINITY;
        if (valid) alpha[base + (size_t)t * Up1 + u] = v;
        // own blank edges (duration >= 1) to diagonal s + k
#pragma unroll
        for (int k = 1; k <= DM; ++k)
          if ((dmask >> k) & 1u) fut[k] = log_add_exp(fut[k], v + o.bl + o.dl[k]);
#pragma unroll
        for (int k = 0; k <= DM; ++k) X(s & 1, k, u) = v + o.ll + o.dl[k];
#pragma unroll
        for (int k = 0; k < DM; ++k) fut[k] = fut[k + 1];
        fut[DM] = -INFINITY;
        __syncthreads();
      }
    }
  } else {
    float hist[DM + 2];   // this thread's beta on diagonal s + k (k >= 1)
#pragma unroll
    for (int k = 0; k < DM + 2; ++k) hist[k] = -INFINITY;
    if (u == Ub) hist[1] = 0.f;           // the virtual cell after the final blank
#pragma unroll
    for (int k = 0; k < DM + 2; ++k) X(1, k, u) = hist[k];
    __syncthreads();
    for (int i0 = 0; i0 < nsteps; i0 += P) {
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const int step = i0 + i;
        if (step >= nsteps) break;        // uniform across the block
        const TdtOps<DM> o = ops[i];
        tdt_operands<DM>(ops[i], step + P < nsteps, cell_t(step + P), u, Tb, Ub, Up1, base, plane, dmask, blank_lp,
                         label_lp, dur_lp);
        const int t = cell_t(step);
        const bool valid = u <= Ub && t >= 0 && t < Tb;
        // the cell's edge terms (blank eb[k], label el[k]) against one shared
        // maximum: one exp2 per term and one log per sum needed (PB, PL, each
        // duration's q, beta) instead of a log-add-exp per term and sum; a
        // term that underflows against the maximum would vanish from every
        // posterior anyway
        float eb[DM + 1], el[DM + 1];
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k <= DM; ++k) {
          // thread u+1's beta on diagonal s + k + 1, i.e. at (t + k, u + 1)
          const float nb = u + 1 < nth ? X((step + 1) & 1, k + 1, u + 1) : -INFINITY;
          eb[k] = k >= 1 ? o.bl + o.dl[k] + hist[k] : -INFINITY;
          el[k] = (u < Ub && t + k < Tb) ? o.ll + o.dl[k] + nb : -INFINITY;
          mx = fmaxf(mx, fmaxf(eb[k], el[k]));
        }
        const bool none = mx == -INFINITY;        // no edge leaves the cell: everything -inf
        const float mk = none ? 0.f : mx * kLog2eDp;
        float sb = 0.f, sl = 0.f, qk[DM + 1];
#pragma unroll
        for (int k = 0; k <= DM; ++k) {
          const float xb = ex2_dp(fmaf(eb[k], kLog2eDp, -mk));   // 0 for -inf terms
          const float xl = ex2_dp(fmaf(el[k], kLog2eDp, -mk));
          sb += xb;
          sl += xl;
          qk[k] = none ? -INFINITY : mx + lg2_dp(xb + xl) * kLn2Dp;
        }
        const float pb = none ? -INFINITY : mx + lg2_dp(sb) * kLn2Dp;
        const float pl = none ? -INFINITY : mx + lg2_dp(sl) * kLn2Dp;
        const float bt = none ? -INFINITY : mx + lg2_dp(sb + sl) * kLn2Dp;
        if (valid) {
          const size_t c = base + (size_t)t * Up1 + u;
          beta_b[c] = pb;
          beta_l[c] = pl;
          int j = 0;
#pragma unroll
          for (int k = 0; k <= DM; ++k)
            if ((dmask >> k) & 1u) {
              q[(size_t)j * plane + c] = qk[k];
              ++j;
            }
          if (t == 0 && u == 0) loss[b] = -bt;
        }
#pragma unroll
        for (int k = DM + 1; k >= 2; --k) hist[k] = hist[k - 1];
        hist[1] = valid ? bt : -INFINITY;
#pragma unroll
        for (int k = 0; k < DM + 2; ++k) X(step & 1, k, u) = hist[k];
        __syncthreads();
      }
    }
  }
}

template <int DM>
void launch_tdt_dp_t(const Shape& s, const Lattice& L, const int32_t* T_len, const int32_t* U_len, float* loss,
                     int threads, cudaStream_t st) {
  dim3 grid(s.B, 2);
  const int smem = 2 * (DM + 2) * threads * (int)sizeof(float);   // <= 80 KB (DM 8, 1024 threads)
  static bool attr[kDeviceSlots] = {};
  const int dev = current_device();
  if (!attr[dev]) {
    cudaFuncSetAttribute(tdt_dp_kernel<DM, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * (DM + 2) * 256 * 4);
    cudaFuncSetAttribute(tdt_dp_kernel<DM, 512>, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * (DM + 2) * 512 * 4);
    cudaFuncSetAttribute(tdt_dp_kernel<DM, 1024>, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * (DM + 2) * 1024 * 4);
    attr[dev] = true;
  }
  if (threads <= 256)
    launch_k(tdt_dp_kernel<DM, 256>, dim3(grid), dim3(threads), smem, st, 1, s.T, s.U, s.dmask, L.plane, L.blank_lp, L.label_lp, L.dur_lp,
                                                        L.alpha, L.beta, L.beta_l, L.tdt_q, T_len, U_len, loss);
  else if (threads <= 512)
    launch_k(tdt_dp_kernel<DM, 512>, dim3(grid), dim3(threads), smem, st, 1, s.T, s.U, s.dmask, L.plane, L.blank_lp, L.label_lp, L.dur_lp,
                                                        L.alpha, L.beta, L.beta_l, L.tdt_q, T_len, U_len, loss);
  else
    launch_k(tdt_dp_kernel<DM, 1024>, dim3(grid), dim3(threads), smem, st, 1, s.T, s.U, s.dmask, L.plane, L.blank_lp, L.label_lp,
                                                         L.dur_lp, L.alpha, L.beta, L.beta_l, L.tdt_q, T_len, U_len,
                                                         loss);
}

void launch_dp_weights(const Shape& s, const Lattice& L, const int32_t* T_len, const int32_t* U_len,
                       cudaStream_t st) {
  if (!L.dpw) return;
  const int threads = ((s.Up1 + 31) / 32) * 32;
  const int NS = dp2_weight_steps(s.T, s.U);
  const long long n = (long long)s.B * 2 * NS * threads;
  const int wb = (int)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  launch_k(dp2_weights_kernel, dim3(wb), dim3(256), 0, st, 1, s.B, s.T, s.U, NS, threads, L.blank_lp, L.label_lp, T_len, U_len, L.dpw);
  note_launch();
}

void launch_dp(const Shape& s, const Lattice& L, const int32_t* T_len, const int32_t* U_len, const int32_t* bounds,
               float* loss, cudaStream_t st) {
  int threads = ((s.Up1 + 31) / 32) * 32;
  if (s.n_dur > 0) {
    switch (s.dmax) {
      case 1: launch_tdt_dp_t<1>(s, L, T_len, U_len, loss, threads, st); break;
      case 2: launch_tdt_dp_t<2>(s, L, T_len, U_len, loss, threads, st); break;
      case 3: launch_tdt_dp_t<3>(s, L, T_len, U_len, loss, threads, st); break;
      case 4: launch_tdt_dp_t<4>(s, L, T_len, U_len, loss, threads, st); break;
      case 5: launch_tdt_dp_t<5>(s, L, T_len, U_len, loss, threads, st); break;
      case 6: launch_tdt_dp_t<6>(s, L, T_len, U_len, loss, threads, st); break;
      case 7: launch_tdt_dp_t<7>(s, L, T_len, U_len, loss, threads, st); break;
      default: launch_tdt_dp_t<8>(s, L, T_len, U_len, loss, threads, st); break;
    }
  } else if (s.S > 0) {
    const int smem = s.T * 4 * (L.path ? 2 : 1);
    if (smem <= 48 * 1024) {
      dim3 grid(s.B, L.path ? 1 : 2);
      const int sp = s.S <= 4 ? 4 : s.S <= 8 ? 8 : s.S <= 16 ? 16 : 32;
      auto kern = sp == 4 ? dp_band_warp_kernel<4> : sp == 8 ? dp_band_warp_kernel<8>
                : sp == 16 ? dp_band_warp_kernel<16> : dp_band_warp_kernel<32>;
      launch_k(kern, dim3(grid), dim3(32), smem, st, 1, s.T, s.U, s.S, bounds, L.blank_lp, L.label_lp, L.alpha, L.beta,
                                                  L.path, T_len, U_len, loss);
    } else {
      launch_k(dp_band_kernel, dim3(s.B), dim3(32), 0, st, 1, s.T, s.U, s.S, bounds, L.blank_lp, L.label_lp, L.alpha, L.beta, L.path,
                                         T_len, U_len, loss);
    }
  } else if (L.path) {
    // decision bits in shared memory when they fit in 96 KB
    const long long words = ((long long)s.T * s.Up1 + 31) / 32;
    const int smem = words * 4 <= 96 * 1024 ? (int)(words * 4) : 0;
    static bool attr[kDeviceSlots] = {};
    const int dev = current_device();
    if (!attr[dev]) {
      cudaFuncSetAttribute(dp_viterbi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
      attr[dev] = true;
    }
    launch_k(dp_viterbi_kernel, dim3(s.B), dim3(threads), smem, st, 1, s.T, s.U, L.blank_lp, L.label_lp, L.alpha, L.path, T_len,
                                                  U_len, loss, smem > 0 ? 1 : 0);
  } else {
    dim3 grid(s.B, 2);
    if (L.dpw)
      launch_k(dp2_kernel<true>, dim3(grid), dim3(threads), 0, st, 1, s.T, s.U, dp2_weight_steps(s.T, s.U), L.blank_lp, L.label_lp, L.dpw,
                                                 L.alpha, L.beta, T_len, U_len, loss);
    else
      launch_k(dp2_kernel<false>, dim3(grid), dim3(threads), 0, st, 1, s.T, s.U, 0, L.blank_lp, L.label_lp, nullptr, L.alpha, L.beta,
                                                  T_len, U_len, loss);
  }
  note_launch();
}

}  // namespace frnnt
