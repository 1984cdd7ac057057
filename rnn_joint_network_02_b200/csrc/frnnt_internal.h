// Internal launcher interface of the frnnt library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "frnnt.h"

namespace frnnt {

// ---------------------------------------------------------------- tracing
// Every launcher calls note_launch() once per kernel it launches; a StageScope
// names the step of the path those launches belong to and, when timing is
// on, brackets it with CUDA events on the stream.
void note_launch(int n = 1);
class StageScope {
 public:
  StageScope(const char* name, cudaStream_t st);
  ~StageScope();
  StageScope(const StageScope&) = delete;
  StageScope& operator=(const StageScope&) = delete;

 private:
  cudaStream_t st_;
  long long launches0_;
  int stage_ = 0;
  cudaEvent_t start_ = nullptr;
};

// ---------------------------------------------------------------- launch chaining
// Programmatic dependent launch.  The kernels of one call follow each other on
// its stream; a kernel launched with the programmatic-serialization attribute
// is launched once the last CTA of the one before it exits, without waiting
// for that grid's completion to be processed, and its CTAs do their set-up
// (barrier init, TMEM allocation, descriptor prefetch) meanwhile (measured:
// tiled call 1.84 -> 1.76 ms, untiled 1.50 -> 1.49 ms on the medium workload).
// So every kernel of the tensor-core path calls chain_wait()
// before it reads or writes memory that an earlier launch of the call writes
// or still reads.  Launched without the attribute, it returns at once.  (No
// kernel triggers its dependents early: a dependent whose CTAs sat resident
// beside a running GEMM, waiting, slowed the tiled call by 30 %.)
__device__ __forceinline__ void chain_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// The call's device-built tile count, read before chain_wait, from L2 (the
// point of coherence), only so that a launch with no tiles in its range can
// skip its set-up.  The prologue that writes the count is complete by then:
// every launch waits for the one before it, also when it has no work, so when
// a launch starts all launches but the previous one have completed, and the
// prologue is at least three launches before any reader of the count.
__device__ __forceinline__ int tile_count_early(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Host side (per host thread): a call names its stream (chain_begin); a kernel
// launched there right after another of the call's kernels gets the attribute;
// any other operation queued on that stream in between (an event record or
// wait) breaks the chain (chain_break), as does the call's end.
void chain_begin(cudaStream_t st);
void chain_break(cudaStream_t st);
void chain_end();
bool chain_take(cudaStream_t st);   // launch with the attribute?
void chain_note(cudaStream_t st);   // a kernel was launched on st

// Launches kern on st (a cluster of cluster_x CTAs when > 1), chained to the
// previous launch where chain_take allows.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  unsigned n = 0;
  if (cluster_x > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster_x;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  if (chain_take(st)) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  chain_note(st);
  return e;
}

// Problem sizes as the launchers see them.
struct Shape {
  int B, T, U, Dx, Dy, H, V, blank;
  int Up1;            // U + 1
  long long BT;       // B * T        (rows of f, F, dF, df)
  long long BU;       // B * (U + 1)  (rows of g, G, dG, dg)
  long long Np;       // B * T * (U + 1) padded lattice cells
  bool bf16;
  bool viterbi;       // maximum-approximation loss
  int S;              // pruned lattice: label positions kept per frame (0 = the whole lattice)
  long long Nlat;     // entries of one lattice array: B*T*(U+1), or B*T*S when pruned
  // token-and-duration transducer (n_dur > 0): the duration set as a bit mask
  // (bit k = duration k frames), its largest entry, and Vx = V + 128: the
  // columns of [W_o; W_d; 0] and the row stride of the logit buffers, whose
  // columns V .. V+n_dur-1 carry the duration head
  int n_dur = 0;
  uint32_t dmask = 0;
  int dmax = 0;
  int Vx = 0;
};

// Lattice arrays, fp32, padded layout [b][t][u] with u fastest.
struct Lattice {
  float* lse;
  float* blank_lp;
  float* label_lp;
  float* alpha;
  float* beta;
  // Maximum approximation only (null otherwise): per cell, bit 0 = the best
  // alignment leaves the cell by its blank edge, bit 1 = by its label edge,
  // bit 2 = the best way into the cell is its blank edge (DP decision).
  uint8_t* path;
  // Token-and-duration transducer only (null otherwise).  beta then holds
  // PB(c) = log of the weight of finishing from c through one of its blank
  // edges, beta_l the same through its label edges (beta(c) = lae(PB, PL));
  // dur_lp [n_dur][plane] the duration log-probs and tdt_q [n_dur][plane]
  // the log posterior numerator of each duration at c without alpha and log P.
  float* beta_l = nullptr;
  float* dur_lp = nullptr;
  float* tdt_q = nullptr;
  long long plane = 0;
  // the two-diagonal DP's precomputed step weights (marginal loss on the
  // whole lattice): dp2_weight_floats(s) floats, else null
  float* dpw = nullptr;
};

// Steps (with the prefetch margin) and floats of the two-diagonal DP's weights.
constexpr int kDp2Prefetch = 4;   // steps the two-diagonal DP loads ahead
inline int dp2_weight_steps(int T, int U) { return (T + U) / 2 + 1 + kDp2Prefetch; }
inline long long dp2_weight_floats(int B, int T, int U) {
  return (long long)B * 2 * dp2_weight_steps(T, U) * 5 * (((U + 1 + 31) / 32) * 32);
}

#ifdef __CUDACC__
// Posterior of the two edges leaving valid cell (t, u) at lattice index c
// (c0 = index of the utterance's cell (0, 0); c_t1 / c_u1 = index of (t+1, u)
// / (t, u+1), or -1 where that cell is not in the lattice; `last` marks
// (T_len-1, U_len), whose blank edge ends the alignment):
//   marginal: bpost = exp(alpha + blank_lp + beta'(t+1,u) - logP) with
//             beta' = 0 after the last cell; lpost = exp(alpha + label_lp + beta(t,u+1) - logP);
//   maximum approximation: the best alignment's 0/1 edge indicators.
__device__ __forceinline__ void edge_posteriors(const Lattice& L, size_t c, size_t c0, long long c_t1,
                                                long long c_u1, bool last, float& bpost, float& lpost) {
  if (L.beta_l) {
    // token-and-duration transducer: the summed posteriors of the blank and
    // of the label edges of every duration, with log P = lae(PB, PL) at (0,0)
    const float x = L.beta[c0], y = L.beta_l[c0];
    const float m = fmaxf(x, y);
    const float logp = m + __logf(__expf(x - m) + __expf(y - m));
    const float al = L.alpha[c] - logp;
    bpost = __expf(al + L.beta[c]);
    lpost = __expf(al + L.beta_l[c]);
    return;
  }
  if (L.path) {
    const uint8_t e = L.path[c];
    bpost = (e & 1) ? 1.f : 0.f;
    lpost = (e & 2) ? 1.f : 0.f;
    return;
  }
  const float logp = L.beta[c0];
  const float al = L.alpha[c];
  const float beta_t1 = c_t1 >= 0 ? L.beta[c_t1] : (last ? 0.f : -INFINITY);
  bpost = __expf(al + L.blank_lp[c] + beta_t1 - logp);
  lpost = c_u1 >= 0 ? __expf(al + L.label_lp[c] + L.beta[c_u1] - logp) : 0.f;
}
#endif

// ---------------------------------------------------------------- validation / DP
void launch_validate(const Shape& s, const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                     const int32_t* bounds, int32_t* status, cudaStream_t st);
void launch_validate_bounds(const Shape& s, const int32_t* bounds, const int32_t* T_len, const int32_t* U_len,
                            int32_t* status, cudaStream_t st);
// The two-diagonal DP's step weights (when L.dpw is set); must precede launch_dp.
void launch_dp_weights(const Shape& s, const Lattice& L, const int32_t* T_len, const int32_t* U_len,
                       cudaStream_t st);
// bounds: the pruned lattice's per-frame starts (s.S > 0), else null
void launch_dp(const Shape& s, const Lattice& L, const int32_t* T_len, const int32_t* U_len, const int32_t* bounds,
               float* loss, cudaStream_t st);

// ---------------------------------------------------------------- CUDA-core kernels
// C[M,N] (fp32, row stride ldc) = op(A)[M,K] * op(B)[K,N]  (+ C when accumulate)
// op(A)(m,k) = transA ? A[k*lda+m] : A[m*lda+k]; op(B)(k,n) = transB ? B[n*ldb+k] : B[k*ldb+n]
// a_bf16 / b_bf16 select the element type of A / B (bf16 or fp32).
void launch_gemm_simt(int M, int N, int K, const void* A, int lda, bool a_bf16, bool transA, const void* B,
                      int ldb, bool b_bf16, bool transB, float* C, int ldc, bool accumulate, cudaStream_t st);

// h[c,:] = tanh(F[b,t,:] + G[b,u,:]) for padded cells c in [c0, c0+C); 0 outside the valid lattice.
void launch_hidden_simt(const Shape& s, const float* F, const float* G, const int32_t* T_len,
                        const int32_t* U_len, long long c0, long long C, float* h, cudaStream_t st);

// z rows of cells [c0, c0+C): z += b_o, then per-cell lse / blank_lp / label_lp into the lattice.
void launch_lse_simt(const Shape& s, float* z, const void* b_o, const int32_t* labels, const int32_t* T_len,
                     const int32_t* U_len, long long c0, long long C, const Lattice& L, cudaStream_t st);

// In place z -> dz for cells [c0, c0+C) (adding b_o first when add_bias); accumulates db_o.
void launch_dz_simt(const Shape& s, float* z, bool add_bias, const void* b_o, const int32_t* labels,
                    const int32_t* T_len, const int32_t* U_len, const float* grad_loss, long long c0,
                    long long C, const Lattice& L, float* db_o_acc, cudaStream_t st);

// dpre = dh * (1 - h^2); dF[b,t] = sum_u dpre (rows of the chunk), dG[b,u] += sum_t dpre.
void launch_dtanh_reduce_simt(const Shape& s, const float* dh, const float* h, long long c0, long long C,
                              float* dF, float* dG, cudaStream_t st);

// ---------------------------------------------------------------- tensor-core GEMM
// D[M,N] = A[M,K] * B[K,N] in bf16 with fp32 accumulation (tcgen05, TMA).
// A: K-major [M][lda] or MN-major [K][lda]; B: K-major [N][ldb] or MN-major [K][ldb].
enum GemmEpilogue { GEMM_EPI_STORE_F32 = 0, GEMM_EPI_STORE_BF16 = 1, GEMM_EPI_RED_F32 = 2, GEMM_EPI_DTANH = 3,
                    GEMM_EPI_DTANH_FG = 4, GEMM_EPI_DTANH_SEG = 5 };

// Lattice cells behind the rows of a GEMM whose 128-row M tiles are cell tiles
// (row m of the GEMM = row m % 128 of cell tile tile0 + m / 128), for the
// d_hidden epilogue that recomputes h = tanh(F[t] + G[u]) instead of reading it.
struct CellMap {
  const int4* tiles = nullptr;    // (b, t0, u0, -)
  int tile0 = 0;
  int T = 0, U = 0, H = 0, UB = 0, S = 0;
  const int32_t* bounds = nullptr;
  const int32_t* T_len = nullptr;
  const int32_t* U_len = nullptr;
  const void* F = nullptr;        // [B*T][H] bf16
  const void* G = nullptr;        // [B*(U+1)][H] bf16
  float* dF = nullptr;            // GEMM_EPI_DTANH_SEG: [B*T][H] fp32, += sum over each frame's cells
  float* dG = nullptr;            //                     [B*(U+1)][H] fp32, += sum over each label position's cells
};
struct GemmTcArgs {
  int M, N, K;
  const void* A;
  bool a_mn;
  long long lda;
  const void* B;
  bool b_mn;
  long long ldb;
  long long b_inner;   // MN-major B: columns of B that hold data (0: N); TMA reads the rest as zeros
  int epi;             // GemmEpilogue
  int k_splits;        // > 1 only with GEMM_EPI_RED_F32; 0 with it: chosen for the launch's rounds
  float* out_f32;      // STORE_F32 / RED_F32 output [M][ldo]
  void* out_bf16;      // STORE_BF16 output, or DTANH h-in / dpre-out [M][ldo]
  long long ldo;
  int32_t* status;     // device status word (timeout bit), may be NULL
  // Optional device-side limit: the effective M (dyn_dim 1) or K (dyn_dim 2)
  // is min(static, (*dyn_count - dyn_base) * dyn_scale), read by the kernel.
  const int* dyn_count = nullptr;
  int dyn_base = 0, dyn_scale = 0, dyn_dim = 0;
  int variant = -1;    // -1 auto, 0 one CTA per tile (M = 128), 1 CTA pairs (M = 256, cta_group::2);
                       // 2 / 3: as 0 / 1 with 256-wide N tiles also for N not a multiple of 256
  CellMap cells;       // GEMM_EPI_DTANH_FG: out = acc * (1 - h^2), h recomputed from F and G;
                       // GEMM_EPI_DTANH_SEG: the same dpre summed into cells.dF / cells.dG, nothing stored
};
int gemm_tc(const GemmTcArgs& g, cudaStream_t st);
// Test setting: the next n gemm_tc launches each drop their CTAs' first K block
// load (so a bounded wait expires and the status word gets FRNNT_STATUS_TIMEOUT);
// returns the previous count.  Process-wide, not thread-safe.
int lose_gemm_loads(int n);
// K slices of a split-K GEMM (frnnt_gemm_tc.cu): mn output tiles on `workers`
// persistent CTAs or CTA pairs, kblocks 64-wide K blocks.
int auto_splits(int mn, int workers, int kblocks);

bool make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_elems,
                       uint32_t box_inner, uint32_t box_outer);

// ---------------------------------------------------------------- fused joint (tensor cores)
struct JointLaunch {
  Shape s;
  int TB, UB;                   // tile = TB frames x UB label positions (TB * UB = 128)
  int mode;                     // 0 forward (lse / blank / label), 1 forward + store z and h, 2 backward dz
  const void* F;                // [B*T][H] bf16
  const void* G;                // [B*(U+1)][H] bf16
  const void* W_o;              // [V][H] bf16
  const void* b_o;              // [V] bf16
  const int32_t* labels;
  const int32_t* T_len;
  const int32_t* U_len;
  const float* grad_loss;
  const int4* tiles;            // device tile list (b, t0, u0, -)
  const int* ntiles;            // device tile count
  int tile_begin, tile_end;     // tile range of this launch (end clamped by *ntiles)
  Lattice L;
  void* zbuf;                   // z (mode 1, rows tile*128+r) or dz (mode 2, rows (tile-begin)*128+r), bf16 [.][V]
  void* hbuf;                   // h rows, same indexing, bf16 [.][hidden_stride(H)]; column H is 1 (cell count column)
  float* db_part;               // unused
  int32_t* status;
  const int32_t* bounds;        // pruned lattice (s.S > 0): [B][T] first label position of each frame's band
  int store_h = 0;              // modes 1 and 2: the generators also write the h rows of hbuf
  const float4* row_params = nullptr;   // mode 2: per-row scalars of the launch's tiles (launch_row_params)
};
bool joint_tc_supported(int H, int V, int T, int U, int S);
// Row stride of the h buffer (H hidden columns, then the [1, 0, ...] column block), padded so the
// dW_o GEMM's N is a whole number of its N tiles.
// Per-device slots of the host-side state that CUDA keeps per device (kernel
// attributes, occupancy answers): a process may drive several GPUs.
constexpr int kDeviceSlots = 64;
inline int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kDeviceSlots) d = 0;
  return d;
}

inline int hidden_stride(int H) { return H >= 512 ? ((H + 1 + 255) / 256) * 256 : ((H + 1 + 127) / 128) * 128; }
void tile_shape(int T, int U, int* TB, int* UB);
// Cell tile of the shape: TB frames x UB label positions, or for a pruned
// lattice TB frames x (S rounded up to a power of two) band positions.
void tile_shape_of(const Shape& s, int* TB, int* UB);
long long max_tiles(const Shape& s, int TB, int UB);
// Regions of fp32 accumulators to clear (16-byte aligned, a multiple of 4 floats each).
struct ZeroList {
  float* ptr[8];
  long long n[8];
  int count;
};
// One launch: the length / label validation (status bits), the tile list and
// the clearing of the accumulators in `z`.
void launch_prologue(const Shape& s, int TB, int UB, const int32_t* labels, const int32_t* T_len,
                     const int32_t* U_len, int32_t* status, int4* tiles, int* ntiles, const ZeroList& z,
                     cudaStream_t st);
int launch_joint_tc(const JointLaunch& j, cudaStream_t st);
// Joint kernel variant for later calls: -1 automatic, 0 one CTA per cell tile, 1 CTA pairs; returns the previous one.
int set_joint_variant(int variant);
void launch_dz_from_z(const JointLaunch& j, cudaStream_t st);
// Token-and-duration transducer: the duration-head logit gradient of the
// launch's rows into columns [V, V + 128) of their dz rows (zeros past n_dur
// and for cells outside the lattice); rows (tile - tile_begin) * 128 + r.
void launch_tdt_dzd(const JointLaunch& j, cudaStream_t st);
// W_x = [W_o; W_d; 0] [Vx][H] and b_x = [b_o; b_d; 0] [Vx] (bf16).
void launch_tdt_weights(const Shape& s, const void* W_o, const void* b_o, const void* W_d, const void* b_d, void* W_x,
                        void* b_x, cudaStream_t st);
// blocks_per_sm: 256-thread blocks per SM of the row-by-row kernel (pruned lattice); the whole
// lattice's tile-by-tile kernel sizes its own grid (up to 6 blocks per SM, as its shared memory allows)
void launch_hidden_rows(const JointLaunch& j, int row_tile0, cudaStream_t st, int blocks_per_sm = 8);
// dW_o = acc[:, :H]; db_o = db (when non-null) or acc[:, H]; acc rows of hidden_stride(H)
void launch_wo_finalize(const float* acc, int V, int H, void* dW_o, void* db_o, cudaStream_t st,
                        const float* db = nullptr, bool out_f32 = false);
// Untiled dz pass that also sums db_o into db_acc [V] (cleared beforehand), for
// dz_db_supported(V, H): the dW_o GEMM then runs on N = H.
bool dz_db_supported(int V, int H);
// Per-row scalars (lse log2 e, w bpost, w lpost, label or -2 for no cell) of
// the tiles [j.tile_begin, j.tile_end), rows (tile - tile_begin) * 128 + r.
void launch_row_params(const JointLaunch& j, float4* row_params, cudaStream_t st);
// row_params: scratch of one float4 per row of the launch's tiles.
void launch_dz_db(const JointLaunch& j, float* db_acc, float4* row_params, cudaStream_t st);

// out[i] = (dtype) in[i]
void launch_convert(const float* in, void* out, long long n, bool to_bf16, cudaStream_t st);
void launch_convert_bf16(const float* in, void* out, long long n, cudaStream_t st);

}  // namespace frnnt
