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
// diagonal, passed by a warp shuffle, and across a warp boundary by a
// parity-double-buffered shared-memory slot.  One block per (utterance,
// direction): alpha and beta run concurrently.
#include "frnnt_common.cuh"
#include "frnnt_internal.h"

namespace frnnt {

__global__ void validate_kernel(int B, int T, int U, int V, int blank, const int32_t* __restrict__ labels,
                                const int32_t* __restrict__ T_len, const int32_t* __restrict__ U_len,
                                int32_t* __restrict__ status) {
  int bits = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    int tl = T_len[b], ul = U_len[b];
    if (tl < 1 || tl > T || ul < 0 || ul > U) bits |= FRNNT_STATUS_LENGTH;
  }
  long long n = (long long)B * U;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) {
    int b = (int)(i / U), u = (int)(i % U);
    int tl = T_len[b], ul = U_len[b];
    if (tl < 1 || tl > T || ul < 0 || ul > U) continue;   // length already flagged
    if (u >= ul) continue;                                // padding label
    int y = labels[i];
    if (y < 0 || y >= V || y == blank) bits |= FRNNT_STATUS_LABEL;
  }
  bits = __reduce_or_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0 && bits) atomicOr(status, bits);
}

void launch_validate(const Shape& s, const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                     int32_t* status, cudaStream_t st) {
  validate_kernel<<<1, 256, 0, st>>>(s.B, s.T, s.U, s.V, s.blank, labels, T_len, U_len, status);
  note_launch();
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

__global__ void dp_kernel(int T, int U, const float* __restrict__ blank_lp, const float* __restrict__ label_lp,
                          float* __restrict__ alpha, float* __restrict__ beta, const int32_t* __restrict__ T_len,
                          const int32_t* __restrict__ U_len, float* __restrict__ loss) {
  __shared__ float xs[2][32];
  const int b = blockIdx.x;
  const bool is_beta = blockIdx.y == 1;
  const int u = threadIdx.x;
  const int lane = u & 31, warp = u >> 5, nwarps = blockDim.x >> 5;
  const Lengths l = lengths_of(T_len, U_len, b, T, U);
  const int Tb = l.Tb, Ub = l.Ub;
  const int Up1 = U + 1;
  const size_t base = (size_t)b * T * Up1;
  const int ndiag = Tb + Ub;        // diagonals d = 0 .. Tb-1+Ub

  float qb[kPrefetch], ql[kPrefetch];
#pragma unroll
  for (int i = 0; i < kPrefetch; ++i)
    dp_operands(is_beta, i, ndiag, u, Tb, Ub, Up1, base, blank_lp, label_lp, qb[i], ql[i]);

  float cur = -INFINITY;            // this thread's value on the previous diagonal
  for (int step0 = 0; step0 < ndiag; step0 += kPrefetch) {
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) {
      const int step = step0 + i;
      if (step >= ndiag) break;     // uniform across the block
      const float ob = qb[i], ol = ql[i];
      dp_operands(is_beta, step + kPrefetch, ndiag, u, Tb, Ub, Up1, base, blank_lp, label_lp, qb[i], ql[i]);
      const int d = is_beta ? (ndiag - 1 - step) : step;
      const int t = d - u;
      const bool active = (u <= Ub) && (t >= 0) && (t < Tb);
      float nb;                     // neighbour's value on the previous diagonal
      if (!is_beta) {
        nb = __shfl_up_sync(0xffffffffu, cur, 1);
        if (lane == 0) nb = warp > 0 ? xs[(step + 1) & 1][warp - 1] : -INFINITY;
      } else {
        nb = __shfl_down_sync(0xffffffffu, cur, 1);
        if (lane == 31) nb = warp + 1 < nwarps ? xs[(step + 1) & 1][warp + 1] : -INFINITY;
      }
      float v = -INFINITY;
      if (active) {
        const size_t c = base + (size_t)t * Up1 + u;
        if (!is_beta) {
          if (t == 0 && u == 0) {
            v = 0.f;
          } else {
            const float fb = t > 0 ? cur + ob : -INFINITY;   // from (t-1, u)
            const float fl = u > 0 ? nb + ol : -INFINITY;    // from (t, u-1)
            v = log_add_exp(fb, fl);
          }
          alpha[c] = v;
        } else {
          if (t == Tb - 1 && u == Ub) {
            v = ob;
          } else {
            const float bb = t + 1 < Tb ? cur + ob : -INFINITY;    // to (t+1, u)
            const float bl = u < Ub ? nb + ol : -INFINITY;         // to (t, u+1)
            v = log_add_exp(bb, bl);
          }
          beta[c] = v;
          if (t == 0 && u == 0) loss[b] = -v;
        }
      }
      cur = v;
      if (!is_beta) {
        if (lane == 31) xs[step & 1][warp] = cur;
      } else {
        if (lane == 0) xs[step & 1][warp] = cur;
      }
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

void launch_dp(const Shape& s, const Lattice& L, const int32_t* T_len, const int32_t* U_len, float* loss,
               cudaStream_t st) {
  int threads = ((s.Up1 + 31) / 32) * 32;
  if (L.path) {
    // decision bits in shared memory when they fit in 96 KB
    const long long words = ((long long)s.T * s.Up1 + 31) / 32;
    const int smem = words * 4 <= 96 * 1024 ? (int)(words * 4) : 0;
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(dp_viterbi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
      attr = true;
    }
    dp_viterbi_kernel<<<s.B, threads, smem, st>>>(s.T, s.U, L.blank_lp, L.label_lp, L.alpha, L.path, T_len,
                                                  U_len, loss, smem > 0 ? 1 : 0);
  } else {
    dim3 grid(s.B, 2);
    dp_kernel<<<grid, threads, 0, st>>>(s.T, s.U, L.blank_lp, L.label_lp, L.alpha, L.beta, T_len, U_len, loss);
  }
  note_launch();
}

}  // namespace frnnt
