// C ABI of the frnnt library: argument checks, workspace planning and the
// launch sequence of one forward + backward call.
//
// One call per batch ("Flash RNN-T", abstract: comparisons use one backward
// call per batch).  Every launch goes on the caller's stream; nothing is
// allocated and nothing is synchronised.
#include <string.h>

#include <mutex>

#include "frnnt_common.cuh"
#include "frnnt_internal.h"

namespace frnnt {
namespace {

constexpr int kDefaultChunkCells = 65536;
// Tensor-core tiled mode, default chunk: four waves of 128-cell tiles over the
// 148 SMs of a B200 (the backward joint pass runs one CTA per SM, so a chunk of
// whole waves leaves no SM idle in its last wave).
constexpr int kDefaultChunkTiles = 4 * 148;

// Bump allocator over the caller's workspace (256-byte aligned slices).
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* p) : base((char*)p) {}
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~(size_t)255;
    T* p = base ? (T*)(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};

bool dims_ok(const frnnt_dims* d) {
  if (d->B <= 0 || d->T <= 0 || d->U < 0 || d->D_enc <= 0 || d->D_pred <= 0 || d->H <= 0 || d->V <= 0) return false;
  if (d->blank < 0 || d->blank >= d->V) return false;
  if (d->U + 1 > 1024) return false;
  if (d->chunk_cells < 0) return false;
  if (d->prune_S < 0 || d->prune_S > 32) return false;
  if (d->wgrad_f32 != 0 && d->wgrad_f32 != 1) return false;
  if (d->n_dur != 0) {
    // token-and-duration transducer: 0 and 1 frames first, strictly increasing, at most 8 frames
    if (d->n_dur < 2 || d->n_dur > FRNNT_MAX_DURATIONS) return false;
    if (d->durations[0] != 0 || d->durations[1] != 1) return false;
    for (int i = 2; i < d->n_dur; ++i)
      if (d->durations[i] <= d->durations[i - 1]) return false;
    if (d->durations[d->n_dur - 1] > FRNNT_MAX_DURATION) return false;
  }
  return true;
}

bool enums_ok(const frnnt_dims* d) {
  if (d->dtype != FRNNT_F32 && d->dtype != FRNNT_BF16) return false;
  if (d->mode != FRNNT_UNTILED && d->mode != FRNNT_TILED) return false;
  if (d->path != FRNNT_PATH_AUTO && d->path != FRNNT_PATH_SIMT) return false;
  if (d->loss != FRNNT_LOSS_MARGINAL && d->loss != FRNNT_LOSS_VITERBI) return false;
  return true;
}

Shape shape_of(const frnnt_dims* d) {
  Shape s;
  s.B = d->B; s.T = d->T; s.U = d->U; s.Dx = d->D_enc; s.Dy = d->D_pred; s.H = d->H; s.V = d->V;
  s.blank = d->blank;
  s.Up1 = d->U + 1;
  s.BT = (long long)d->B * d->T;
  s.BU = (long long)d->B * (d->U + 1);
  s.Np = s.BT * s.Up1;
  s.bf16 = d->dtype == FRNNT_BF16;
  s.viterbi = d->loss == FRNNT_LOSS_VITERBI;
  s.S = d->prune_S;
  s.Nlat = s.S > 0 ? s.BT * s.S : s.Np;
  s.n_dur = d->n_dur;
  s.dmask = 0;
  s.dmax = 0;
  for (int i = 0; i < d->n_dur; ++i) {
    s.dmask |= 1u << d->durations[i];
    s.dmax = d->durations[i] > s.dmax ? d->durations[i] : s.dmax;
  }
  s.Vx = d->n_dur > 0 ? d->V + 128 : d->V;
  return s;
}

// ------------------------------------------------------------------ SIMT plan
struct SimtPlan {
  float *F, *G, *dF, *dG;
  Lattice L;
  float *accWf, *accWg, *accWo, *accbo;
  float *df_tmp, *dg_tmp;
  float *h, *dh, *z;
  long long rows_per_chunk;
  size_t bytes;
};

SimtPlan plan_simt(const frnnt_dims* d, const Shape& s, void* ws) {
  SimtPlan p;
  Carver c(ws);
  long long cells = d->chunk_cells > 0 ? d->chunk_cells : kDefaultChunkCells;
  p.rows_per_chunk = cells / s.Up1;
  if (p.rows_per_chunk < 1) p.rows_per_chunk = 1;
  if (p.rows_per_chunk > s.BT) p.rows_per_chunk = s.BT;
  const long long C = p.rows_per_chunk * s.Up1;
  p.F = c.take<float>(s.BT * s.H);
  p.G = c.take<float>(s.BU * s.H);
  p.dF = c.take<float>(s.BT * s.H);
  p.dG = c.take<float>(s.BU * s.H);
  p.L.lse = c.take<float>(s.Np);
  p.L.blank_lp = c.take<float>(s.Np);
  p.L.label_lp = c.take<float>(s.Np);
  p.L.alpha = c.take<float>(s.Np);
  p.L.beta = c.take<float>(s.Np);
  p.L.path = s.viterbi ? c.take<uint8_t>(s.Np) : nullptr;
  p.L.dpw = s.viterbi ? nullptr : c.take<float>(dp2_weight_floats(s.B, s.T, s.U));
  p.accWf = c.take<float>((size_t)s.Dx * s.H);
  p.accWg = c.take<float>((size_t)s.Dy * s.H);
  p.accWo = c.take<float>((size_t)s.V * s.H);
  p.accbo = c.take<float>(s.V);
  p.df_tmp = s.bf16 ? c.take<float>(s.BT * s.Dx) : nullptr;
  p.dg_tmp = s.bf16 ? c.take<float>(s.BU * s.Dy) : nullptr;
  p.h = c.take<float>(C * s.H);
  p.dh = c.take<float>(C * s.H);
  p.z = c.take<float>((d->mode == FRNNT_UNTILED ? s.Np : C) * s.V);
  p.bytes = c.off + 256;
  return p;
}

int run_simt(const frnnt_dims* d, const Shape& s, const void* f, const void* g, const void* W_f, const void* W_g,
             const void* W_o, const void* b_o, const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
             const float* grad_loss, float* loss, void* df, void* dg, void* dW_f, void* dW_g, void* dW_o,
             void* db_o, void* ws, int32_t* status, cudaStream_t st) {
  SimtPlan p = plan_simt(d, s, ws);
  const bool bf = s.bf16;
  const bool untiled = d->mode == FRNNT_UNTILED;
  {
    StageScope sc("validate", st);
    launch_validate(s, labels, T_len, U_len, nullptr, status, st);
    cudaMemsetAsync(p.dG, 0, s.BU * s.H * sizeof(float), st);
    cudaMemsetAsync(p.accWo, 0, (size_t)s.V * s.H * sizeof(float), st);
    cudaMemsetAsync(p.accbo, 0, (size_t)s.V * sizeof(float), st);
  }
  {  // projections F = f W_f, G = g W_g
    StageScope sc("projection", st);
    launch_gemm_simt((int)s.BT, s.H, s.Dx, f, s.Dx, bf, false, W_f, s.H, bf, false, p.F, s.H, false, st);
    launch_gemm_simt((int)s.BU, s.H, s.Dy, g, s.Dy, bf, false, W_g, s.H, bf, false, p.G, s.H, false, st);
  }

  // forward joint: per-cell log-sum-exp, blank and label log-probs
  for (long long r0 = 0; r0 < s.BT; r0 += p.rows_per_chunk) {
    StageScope sc("joint_fwd", st);
    const long long nr = (r0 + p.rows_per_chunk <= s.BT) ? p.rows_per_chunk : s.BT - r0;
    const long long c0 = r0 * s.Up1, C = nr * s.Up1;
    float* zc = untiled ? p.z + (size_t)c0 * s.V : p.z;
    launch_hidden_simt(s, p.F, p.G, T_len, U_len, c0, C, p.h, st);
    launch_gemm_simt((int)C, s.V, s.H, p.h, s.H, false, false, W_o, s.H, bf, true, zc, s.V, false, st);
    launch_lse_simt(s, zc, b_o, labels, T_len, U_len, c0, C, p.L, st);
  }

  {  // transducer forward-backward
    StageScope sc("lattice_dp", st);
    launch_dp_weights(s, p.L, T_len, U_len, st);
    launch_dp(s, p.L, T_len, U_len, nullptr, loss, st);
  }

  // backward through the joint
  for (long long r0 = 0; r0 < s.BT; r0 += p.rows_per_chunk) {
    StageScope sc("joint_bwd", st);
    const long long nr = (r0 + p.rows_per_chunk <= s.BT) ? p.rows_per_chunk : s.BT - r0;
    const long long c0 = r0 * s.Up1, C = nr * s.Up1;
    float* zc = untiled ? p.z + (size_t)c0 * s.V : p.z;
    launch_hidden_simt(s, p.F, p.G, T_len, U_len, c0, C, p.h, st);
    if (!untiled) launch_gemm_simt((int)C, s.V, s.H, p.h, s.H, false, false, W_o, s.H, bf, true, zc, s.V, false, st);
    launch_dz_simt(s, zc, !untiled, b_o, labels, T_len, U_len, grad_loss, c0, C, p.L, p.accbo, st);
    launch_gemm_simt((int)C, s.H, s.V, zc, s.V, false, false, W_o, s.H, bf, false, p.dh, s.H, false, st);
    launch_dtanh_reduce_simt(s, p.dh, p.h, c0, C, p.dF, p.dG, st);
    launch_gemm_simt(s.V, s.H, (int)C, zc, s.V, false, true, p.h, s.H, false, false, p.accWo, s.H, true, st);
  }

  StageScope sc("projection_bwd", st);
  float* dfo = bf ? p.df_tmp : (float*)df;
  float* dgo = bf ? p.dg_tmp : (float*)dg;
  launch_gemm_simt((int)s.BT, s.Dx, s.H, p.dF, s.H, false, false, W_f, s.H, bf, true, dfo, s.Dx, false, st);
  launch_gemm_simt(s.Dx, s.H, (int)s.BT, f, s.Dx, bf, true, p.dF, s.H, false, false, p.accWf, s.H, false, st);
  launch_gemm_simt((int)s.BU, s.Dy, s.H, p.dG, s.H, false, false, W_g, s.H, bf, true, dgo, s.Dy, false, st);
  launch_gemm_simt(s.Dy, s.H, (int)s.BU, g, s.Dy, bf, true, p.dG, s.H, false, false, p.accWg, s.H, false, st);
  if (bf) {
    launch_convert(p.df_tmp, df, s.BT * s.Dx, true, st);
    launch_convert(p.dg_tmp, dg, s.BU * s.Dy, true, st);
  }
  const bool wbf = bf && !d->wgrad_f32;   // weight gradients rounded to bf16, or the fp32 accumulators
  launch_convert(p.accWf, dW_f, (long long)s.Dx * s.H, wbf, st);
  launch_convert(p.accWg, dW_g, (long long)s.Dy * s.H, wbf, st);
  launch_convert(p.accWo, dW_o, (long long)s.V * s.H, wbf, st);
  launch_convert(p.accbo, db_o, s.V, wbf, st);
  return cudaGetLastError() == cudaSuccess ? FRNNT_OK : FRNNT_ERR_CUDA;
}


// ------------------------------------------------------------------ tensor-core plan
bool use_tc(const frnnt_dims* d) {
  if (d->dtype != FRNNT_BF16 || d->path != FRNNT_PATH_AUTO) return false;
  if (d->B > 1024) return false;
  if (d->H % 64 || d->D_enc % 32 || d->D_pred % 32) return false;
  return joint_tc_supported(d->H, d->n_dur > 0 ? d->V + 128 : d->V, d->T, d->U, d->prune_S);
}

// The token-and-duration transducer runs on the tensor-core kernels, with the
// marginal loss, over the whole lattice.
bool tdt_supported(const frnnt_dims* d) {
  return use_tc(d) && d->loss == FRNNT_LOSS_MARGINAL && d->prune_S == 0;
}

struct TcPlan {
  int TB, UB;
  long long maxT, chunkT;
  __nv_bfloat16 *F, *G;
  float *dF, *dG;
  __nv_bfloat16 *dFb, *dGb;
  int4* tiles;
  int* ntiles;
  Lattice L;
  float *accWo, *db_part, *accWf, *accWg;
  __nv_bfloat16 *zbuf, *hbuf;
  // token-and-duration transducer: [W_o; W_d; 0], [b_o; b_d; 0] and the
  // duration head's weight-gradient accumulator (64 rows, n_dur used)
  __nv_bfloat16 *Wx = nullptr, *bx = nullptr;
  float4* row_params = nullptr;   // the dz pass with bias sums: per-row scalars
  float* accWd = nullptr;
  size_t bytes;
};

TcPlan plan_tc(const frnnt_dims* d, const Shape& s, void* ws) {
  TcPlan p;
  Carver c(ws);
  tile_shape_of(s, &p.TB, &p.UB);
  p.maxT = max_tiles(s, p.TB, p.UB);
  p.chunkT = d->chunk_cells > 0 ? (d->chunk_cells + 127) / 128 : kDefaultChunkTiles;
  if (p.chunkT > p.maxT) p.chunkT = p.maxT;
  if (d->mode == FRNNT_UNTILED) p.chunkT = p.maxT;
  p.F = c.take<__nv_bfloat16>(s.BT * s.H);
  p.G = c.take<__nv_bfloat16>(s.BU * s.H);
  p.dF = c.take<float>(s.BT * s.H);
  p.dG = c.take<float>(s.BU * s.H);
  p.tiles = c.take<int4>(p.maxT);
  p.ntiles = c.take<int>(4);
  p.L.lse = c.take<float>(s.Nlat);
  p.L.blank_lp = c.take<float>(s.Nlat);
  p.L.label_lp = c.take<float>(s.Nlat);
  p.L.alpha = c.take<float>(s.Nlat);
  p.L.beta = c.take<float>(s.Nlat);
  p.L.path = s.viterbi ? c.take<uint8_t>(s.Nlat) : nullptr;
  // the two-diagonal DP forms its step weights step by step (no weight
  // array: measured as fast as precomputing them by a parallel pass, which
  // competes with the hidden rows beside the DP in untiled mode)
  p.L.dpw = nullptr;
  if (s.n_dur > 0) {
    p.L.beta_l = c.take<float>(s.Nlat);
    p.L.dur_lp = c.take<float>((size_t)s.n_dur * s.Nlat);
    p.L.tdt_q = c.take<float>((size_t)s.n_dur * s.Nlat);
    p.L.plane = s.Nlat;
    p.Wx = c.take<__nv_bfloat16>((size_t)s.Vx * s.H);
    p.bx = c.take<__nv_bfloat16>(s.Vx);
    p.accWd = c.take<float>((size_t)64 * hidden_stride(s.H));
  }
  p.accWo = c.take<float>((size_t)s.V * hidden_stride(s.H));
  // untiled with H a multiple of 256: db_o is summed by the dz pass, so the
  // dW_o GEMM runs on N = H (whole 256-wide tiles) without the ones column
  p.db_part = (d->mode == FRNNT_UNTILED && dz_db_supported(s.V, s.H)) ? c.take<float>(s.V) : nullptr;
  // per-row scalars of the dz pass: the whole lattice (untiled, with db_o
  // sums) or one chunk (tiled)
  p.row_params = p.db_part ? c.take<float4>((size_t)p.maxT * 128)
                           : (d->mode == FRNNT_TILED ? c.take<float4>((size_t)p.chunkT * 128) : nullptr);
  p.accWf = c.take<float>((size_t)s.Dx * s.H);
  p.accWg = c.take<float>((size_t)s.Dy * s.H);
  const size_t zb = (size_t)p.chunkT * 128 * s.Vx, hb = (size_t)p.chunkT * 128 * hidden_stride(s.H);
  p.zbuf = c.take<__nv_bfloat16>(zb);
  p.hbuf = c.take<__nv_bfloat16>(hb);
  // bf16 copies of dF and dG for the projection backward, made after the last
  // chunk: they reuse the chunk buffers when those are large enough
  const size_t fb = (size_t)s.BT * s.H, gb = (size_t)s.BU * s.H;
  if ((((fb + 127) & ~(size_t)127) + gb) <= zb + hb) {
    p.dFb = p.zbuf;
    p.dGb = p.zbuf ? p.zbuf + ((fb + 127) & ~(size_t)127) : nullptr;
  } else {
    p.dFb = c.take<__nv_bfloat16>(fb);
    p.dGb = c.take<__nv_bfloat16>(gb);
  }
  p.bytes = c.off + 256;
  return p;
}

// A second stream per device for work that runs beside the lattice DP (which
// occupies one block per utterance and direction), forked from and joined
// back to the caller's stream with events, so stream order, graph capture and
// the caller's synchronisation are unaffected.  Shared by all calls on the
// device: between one call's record of `fork` and its stream's wait on it,
// another call's record would redirect that wait.  So a call holds the
// device's `mu` from before its first fork until after its last join wait
// (host-side queuing only; calls on different devices use different slots).
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;     // hidden rows beside the lattice DP
  cudaEvent_t fork2 = nullptr, join2 = nullptr;   // the G-side projection backward beside the F side
  bool ok = false;
  std::mutex mu;
};

SideStream* side_stream() {
  static SideStream sides[64];
  static std::mutex init_mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& x = sides[dev];
  std::lock_guard<std::mutex> guard(init_mu);
  if (!x.ok && !x.s) {
    if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) == cudaSuccess &&
        cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&x.fork2, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&x.join2, cudaEventDisableTiming) == cudaSuccess)
      x.ok = true;
    else
      cudaGetLastError();
  }
  return x.ok ? &x : nullptr;
}

int run_tc(const frnnt_dims* d, const Shape& s, const void* f, const void* g, const void* W_f, const void* W_g,
           const void* W_o, const void* b_o, const void* W_d, const void* b_d, const int32_t* labels,
           const int32_t* T_len, const int32_t* U_len, const int32_t* bounds, const float* grad_loss, float* loss,
           void* df, void* dg, void* dW_f, void* dW_g, void* dW_o, void* db_o, void* dW_d, void* db_d, void* ws,
           int32_t* status, cudaStream_t st) {
  TcPlan p = plan_tc(d, s, ws);
  const bool untiled = d->mode == FRNNT_UNTILED;
  const bool tdt = s.n_dur > 0;
  const bool wf32 = d->wgrad_f32 != 0;
  int rc = FRNNT_OK;
  // the side stream's fork / join events are shared by the device's calls:
  // hold its lock while this call queues work (released on every return)
  SideStream* side_lock = side_stream();
  std::unique_lock<std::mutex> queue_lock;
  if (side_lock) queue_lock = std::unique_lock<std::mutex>(side_lock->mu);
  // consecutive kernels of this call on st are chained (each may start while
  // the one before drains); ended on every return
  struct ChainScope {
    explicit ChainScope(cudaStream_t s) { chain_begin(s); }
    ~ChainScope() { chain_end(); }
  } chain_scope(st);
#define FRNNT_TRY(x)            \
  do {                          \
    rc = (x);                   \
    if (rc != FRNNT_OK) return rc; \
  } while (0)
  {
    StageScope sc("validate", st);
    // validation, tile list and cleared accumulators in one launch
    ZeroList z{};
    auto add = [&](float* ptr, long long n) {
      z.ptr[z.count] = ptr;
      z.n[z.count] = n;
      ++z.count;
    };
    add(p.dF, s.BT * s.H);
    add(p.dG, s.BU * s.H);
    add(p.accWo, (long long)s.V * hidden_stride(s.H));
    add(p.accWf, (long long)s.Dx * s.H);
    add(p.accWg, (long long)s.Dy * s.H);
    if (tdt) add(p.accWd, 64LL * hidden_stride(s.H));
    if (p.db_part) add(p.db_part, (s.V + 3) / 4 * 4);
    launch_prologue(s, p.TB, p.UB, labels, T_len, U_len, status, p.tiles, p.ntiles, z, st);
    if (s.S > 0) launch_validate_bounds(s, bounds, T_len, U_len, status, st);
    if (tdt) launch_tdt_weights(s, W_o, b_o, W_d, b_d, p.Wx, p.bx, st);
  }
  {
    StageScope sc("projection", st);
    GemmTcArgs a{};
    a.M = (int)s.BT; a.N = s.H; a.K = s.Dx; a.A = f; a.a_mn = false; a.lda = s.Dx; a.B = W_f; a.b_mn = true;
    a.ldb = s.H; a.epi = GEMM_EPI_STORE_BF16; a.k_splits = 1; a.out_bf16 = p.F; a.ldo = s.H; a.status = status;
    FRNNT_TRY(gemm_tc(a, st));
    a.M = (int)s.BU; a.K = s.Dy; a.A = g; a.lda = s.Dy; a.B = W_g; a.out_bf16 = p.G;
    FRNNT_TRY(gemm_tc(a, st));
  }
  JointLaunch j{};
  j.s = s; j.TB = p.TB; j.UB = p.UB; j.F = p.F; j.G = p.G; j.W_o = tdt ? (const void*)p.Wx : W_o;
  j.b_o = tdt ? (const void*)p.bx : b_o; j.labels = labels;
  j.T_len = T_len; j.U_len = U_len; j.grad_loss = grad_loss; j.tiles = p.tiles; j.ntiles = p.ntiles; j.L = p.L;
  j.zbuf = p.zbuf; j.hbuf = p.hbuf; j.db_part = p.db_part; j.status = status; j.bounds = bounds;
  // tiled: the backward joint pass (mode 2) also stores the h rows of each
  // chunk (its generators have the time; a separate pass would re-read F and
  // G); untiled: the forward pass already stores z, and a second stream of
  // stores there costs more than the hidden-row kernel beside the DP
  j.store_h = 0;
  {
    StageScope sc("joint_fwd", st);
    j.mode = untiled ? 1 : 0;
    j.tile_begin = 0;
    j.tile_end = (int)p.maxT;
    FRNNT_TRY(launch_joint_tc(j, st));
  }
  {
    // the DP's step weights first: a short full-GPU pass, done before the
    // hidden rows below take the SMs
    StageScope sc("lattice_dp", st);
    launch_dp_weights(s, p.L, T_len, U_len, st);
  }
  // untiled: the h rows of the whole lattice do not depend on the DP; build
  // them on the side stream while the DP runs
  SideStream* side = untiled ? side_stream() : nullptr;
  if (side) {
    j.tile_begin = 0;
    j.tile_end = (int)p.maxT;
    cudaEventRecord(side->fork, st);
    chain_break(st);
    cudaStreamWaitEvent(side->s, side->fork, 0);
    {
      StageScope sc("bwd_hidden", side->s);
      launch_hidden_rows(j, 0, side->s);
    }
    cudaEventRecord(side->join, side->s);
  }
  {
    StageScope sc("lattice_dp", st);
    launch_dp(s, p.L, T_len, U_len, bounds, loss, st);
  }
  for (long long c0 = 0; c0 < p.maxT; c0 += p.chunkT) {
    const long long c1 = (c0 + p.chunkT < p.maxT) ? c0 + p.chunkT : p.maxT;
    j.tile_begin = (int)c0;
    j.tile_end = (int)c1;
    __nv_bfloat16* zrows = untiled ? p.zbuf + (size_t)c0 * 128 * s.Vx : p.zbuf;
    const int HS = hidden_stride(s.H);
    __nv_bfloat16* hrows = untiled ? p.hbuf + (size_t)c0 * 128 * HS : p.hbuf;
    {
      StageScope sc("joint_bwd_dz", st);
      if (untiled) {
        if (p.db_part) launch_dz_db(j, p.db_part, p.row_params, st);
        else launch_dz_from_z(j, st);
      } else {
        j.mode = 2;
        j.store_h = 1;
        j.row_params = p.row_params;
        launch_row_params(j, p.row_params, st);
        FRNNT_TRY(launch_joint_tc(j, st));
        if (tdt) launch_tdt_dzd(j, st);
      }
    }
    const int rows = (int)((c1 - c0) * 128);
    auto run_dWo = [&]() -> int {
      StageScope sc("bwd_dWo", st);
      GemmTcArgs a{};
      // dW_o | db_o = dz^T [h | 1]: the extra column block of h yields the bias
      // gradient, unless the dz pass summed it (then N = H)
      a.M = s.V; a.N = p.db_part ? s.H : HS; a.K = rows; a.A = zrows; a.a_mn = true; a.lda = s.Vx; a.B = hrows;
      a.b_mn = true; a.ldb = HS; a.epi = GEMM_EPI_RED_F32; a.k_splits = 0;
      // tiled: the recompute pass writes h rows up to the column block that
      // holds the 1 of column H; the columns past it are read as zeros
      a.b_inner = untiled ? 0 : s.H + 8;
      a.out_f32 = p.accWo;
      a.ldo = HS; a.status = status; a.dyn_count = p.ntiles; a.dyn_base = (int)c0; a.dyn_scale = 128;
      a.dyn_dim = 2;
      const int r = gemm_tc(a, st);
      if (r != FRNNT_OK || !tdt) return r;
      // dW_d | db_d from the duration columns (64 of them, zero past n_dur)
      a.M = 64; a.N = HS; a.A = zrows + s.V; a.k_splits = 0; a.out_f32 = p.accWd;
      return gemm_tc(a, st);
    };
    auto run_dh = [&]() -> int {
      StageScope sc("bwd_dh", st);
      GemmTcArgs a{};
      // d_hidden = dz W_o; the epilogue forms dpre = d_hidden (1 - h^2), with h
      // recomputed from the L2-resident F and G rows of each cell (not read
      // back), and sums it into dF (per frame) and dG (per label position):
      // dpre is never stored
      // (token-and-duration transducer: dz | dzd against [W_o; W_d], K = V + 64)
      a.M = rows; a.N = s.H; a.K = tdt ? s.V + 64 : s.V; a.A = zrows; a.a_mn = false; a.lda = s.Vx;
      a.B = tdt ? (const void*)p.Wx : W_o; a.b_mn = true; a.ldb = s.H; a.epi = GEMM_EPI_DTANH_SEG; a.k_splits = 1;
      a.status = status;
      a.cells.tiles = p.tiles; a.cells.tile0 = (int)c0; a.cells.T = s.T; a.cells.U = s.U; a.cells.H = s.H;
      a.cells.UB = p.UB; a.cells.S = s.S; a.cells.bounds = bounds; a.cells.T_len = T_len; a.cells.U_len = U_len;
      a.cells.F = p.F; a.cells.G = p.G; a.cells.dF = p.dF; a.cells.dG = p.dG;
      a.dyn_count = p.ntiles; a.dyn_base = (int)c0; a.dyn_scale = 128; a.dyn_dim = 1;
      return gemm_tc(a, st);
    };
    // untiled: d_hidden first (it does not read the h rows, so it need not wait
    // for the side stream; measured 0.03 ms faster on medium and 0.3 ms on
    // long than after dW_o); tiled: dW_o first, while the chunk's last-written
    // dz and h rows are still in L2 (measured 0.01-0.14 ms faster)
    if (untiled) FRNNT_TRY(run_dh());
    if (side) {   // the h rows of the side stream, for dW_o
      cudaStreamWaitEvent(st, side->join, 0);
      chain_break(st);
    } else if (untiled) {   // no side stream could be created: build the h rows here
      StageScope sc("bwd_hidden", st);
      launch_hidden_rows(j, 0, st);
    }
    FRNNT_TRY(run_dWo());
    if (!untiled) FRNNT_TRY(run_dh());
  }
  {
    StageScope sc("projection_bwd", st);
    // the G side (dg, dW_g) runs on the side stream beside the F side (df,
    // dW_f); forked from and joined back to the caller's stream by events
    SideStream* ps = side_stream();
    cudaStream_t gs = ps ? ps->s : st;
    if (ps) {
      cudaEventRecord(ps->fork2, st);
      chain_break(st);
      cudaStreamWaitEvent(gs, ps->fork2, 0);
    }
    launch_wo_finalize(p.accWo, s.V, s.H, dW_o, db_o, st, p.db_part, wf32);
    if (tdt) launch_wo_finalize(p.accWd, s.n_dur, s.H, dW_d, db_d, st, nullptr, wf32);
    launch_convert_bf16(p.dF, p.dFb, s.BT * s.H, st);
    launch_convert_bf16(p.dG, p.dGb, s.BU * s.H, gs);
    GemmTcArgs a{};
    // df = dF W_f^T : B = W_f read as K-major [D_enc][H]
    a.M = (int)s.BT; a.N = s.Dx; a.K = s.H; a.A = p.dFb; a.a_mn = false; a.lda = s.H; a.B = W_f; a.b_mn = false;
    a.ldb = s.H; a.epi = GEMM_EPI_STORE_BF16; a.k_splits = 1; a.out_bf16 = df; a.ldo = s.Dx; a.status = status;
    int rc_f = gemm_tc(a, st);
    a.M = (int)s.BU; a.N = s.Dy; a.A = p.dGb; a.B = W_g; a.out_bf16 = dg; a.ldo = s.Dy;
    int rc_g = gemm_tc(a, gs);
    // dW_f = f^T dF : A = f read as MN-major [BT][D_enc], B = dF MN-major [BT][H]
    GemmTcArgs w{};
    w.M = s.Dx; w.N = s.H; w.K = (int)s.BT; w.A = f; w.a_mn = true; w.lda = s.Dx; w.B = p.dFb; w.b_mn = true;
    w.ldb = s.H; w.epi = GEMM_EPI_RED_F32; w.k_splits = 0; w.out_f32 = p.accWf;
    w.ldo = s.H; w.status = status;
    if (rc_f == FRNNT_OK) rc_f = gemm_tc(w, st);
    w.M = s.Dy; w.K = (int)s.BU; w.A = g; w.lda = s.Dy; w.B = p.dGb; w.k_splits = 0;
    w.out_f32 = p.accWg;
    if (rc_g == FRNNT_OK) rc_g = gemm_tc(w, gs);
    launch_convert(p.accWf, dW_f, (long long)s.Dx * s.H, !wf32, st);
    launch_convert(p.accWg, dW_g, (long long)s.Dy * s.H, !wf32, gs);
    if (ps) {   // joined on every path, so the caller's stream never runs ahead of the side work
      cudaEventRecord(ps->join2, gs);
      cudaStreamWaitEvent(st, ps->join2, 0);
      chain_break(st);
    }
    FRNNT_TRY(rc_f);
    FRNNT_TRY(rc_g);
  }
#undef FRNNT_TRY
  return cudaGetLastError() == cudaSuccess ? FRNNT_OK : FRNNT_ERR_CUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace frnnt

using namespace frnnt;

extern "C" int frnnt_workspace_size(const frnnt_dims* d, size_t* bytes) {
  if (!d || !bytes) return FRNNT_ERR_NULL;
  if (!enums_ok(d)) return FRNNT_ERR_UNSUPPORTED;
  if (!dims_ok(d)) return FRNNT_ERR_DIMS;
  if (d->prune_S > 0 && !use_tc(d)) return FRNNT_ERR_UNSUPPORTED;
  if (d->n_dur > 0 && !tdt_supported(d)) return FRNNT_ERR_UNSUPPORTED;
  Shape s = shape_of(d);
  *bytes = use_tc(d) ? plan_tc(d, s, nullptr).bytes : plan_simt(d, s, nullptr).bytes;
  return FRNNT_OK;
}

namespace {

int fwd_bwd_impl(const frnnt_dims* d, const void* f, const void* g, const void* W_f, const void* W_g, const void* W_o,
                 const void* b_o, const void* W_d, const void* b_d, const int32_t* labels, const int32_t* T_len,
                 const int32_t* U_len, const int32_t* bounds, const float* grad_loss, float* loss, void* df, void* dg,
                 void* dW_f, void* dW_g, void* dW_o, void* db_o, void* dW_d, void* db_d, void* workspace,
                 size_t workspace_bytes, int32_t* status, void* stream) {
  if (!d) return FRNNT_ERR_NULL;
  if (!enums_ok(d)) return FRNNT_ERR_UNSUPPORTED;
  if (!dims_ok(d)) return FRNNT_ERR_DIMS;
  if (d->prune_S > 0 && !use_tc(d)) return FRNNT_ERR_UNSUPPORTED;
  if (d->n_dur > 0 && !tdt_supported(d)) return FRNNT_ERR_UNSUPPORTED;
  const void* req[] = {f, g, W_f, W_g, W_o, b_o, T_len, U_len, loss, df, dg, dW_f, dW_g, dW_o, db_o, workspace, status};
  for (const void* p : req)
    if (!p) return FRNNT_ERR_NULL;
  if (!labels && d->U > 0) return FRNNT_ERR_NULL;
  if (d->prune_S > 0 && !bounds) return FRNNT_ERR_NULL;
  if (d->n_dur > 0 && (!W_d || !b_d || !dW_d || !db_d)) return FRNNT_ERR_NULL;
  const void* al[] = {f, g, W_f, W_g, W_o, b_o, W_d, b_d, labels, T_len, U_len, bounds, grad_loss, loss, df, dg,
                      dW_f, dW_g, dW_o, db_o, dW_d, db_d, workspace, status};
  for (const void* p : al)
    if (p && !aligned16(p)) return FRNNT_ERR_ALIGN;
  size_t need = 0;
  frnnt_workspace_size(d, &need);
  if (workspace_bytes < need) return FRNNT_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  Shape s = shape_of(d);
  cudaGetLastError();   // clear a stale error so it is not reported as ours
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return FRNNT_ERR_CUDA;
  if (use_tc(d))
    return run_tc(d, s, f, g, W_f, W_g, W_o, b_o, W_d, b_d, labels, T_len, U_len, bounds, grad_loss, loss, df, dg,
                  dW_f, dW_g, dW_o, db_o, dW_d, db_d, workspace, status, st);
  return run_simt(d, s, f, g, W_f, W_g, W_o, b_o, labels, T_len, U_len, grad_loss, loss, df, dg, dW_f, dW_g, dW_o,
                  db_o, workspace, status, st);
}

}  // namespace

extern "C" int frnnt_fwd_bwd(const frnnt_dims* d, const void* f, const void* g, const void* W_f, const void* W_g,
                             const void* W_o, const void* b_o, const int32_t* labels, const int32_t* T_len,
                             const int32_t* U_len, const float* grad_loss, float* loss, void* df, void* dg,
                             void* dW_f, void* dW_g, void* dW_o, void* db_o, void* workspace, size_t workspace_bytes,
                             int32_t* status, void* stream) {
  // pruned dims go through frnnt_fwd_bwd_pruned, duration sets through frnnt_fwd_bwd_tdt
  if (d && (d->prune_S != 0 || d->n_dur != 0)) return FRNNT_ERR_DIMS;
  return fwd_bwd_impl(d, f, g, W_f, W_g, W_o, b_o, nullptr, nullptr, labels, T_len, U_len, nullptr, grad_loss, loss,
                      df, dg, dW_f, dW_g, dW_o, db_o, nullptr, nullptr, workspace, workspace_bytes, status, stream);
}

extern "C" int frnnt_fwd_bwd_pruned(const frnnt_dims* d, const void* f, const void* g, const void* W_f,
                                    const void* W_g, const void* W_o, const void* b_o, const int32_t* labels,
                                    const int32_t* T_len, const int32_t* U_len, const int32_t* bounds,
                                    const float* grad_loss, float* loss, void* df, void* dg, void* dW_f, void* dW_g,
                                    void* dW_o, void* db_o, void* workspace, size_t workspace_bytes, int32_t* status,
                                    void* stream) {
  if (d && (d->prune_S <= 0 || d->n_dur != 0)) return FRNNT_ERR_DIMS;
  return fwd_bwd_impl(d, f, g, W_f, W_g, W_o, b_o, nullptr, nullptr, labels, T_len, U_len, bounds, grad_loss, loss,
                      df, dg, dW_f, dW_g, dW_o, db_o, nullptr, nullptr, workspace, workspace_bytes, status, stream);
}

extern "C" int frnnt_fwd_bwd_tdt(const frnnt_dims* d, const void* f, const void* g, const void* W_f, const void* W_g,
                                 const void* W_o, const void* b_o, const void* W_d, const void* b_d,
                                 const int32_t* labels, const int32_t* T_len, const int32_t* U_len,
                                 const float* grad_loss, float* loss, void* df, void* dg, void* dW_f, void* dW_g,
                                 void* dW_o, void* db_o, void* dW_d, void* db_d, void* workspace,
                                 size_t workspace_bytes, int32_t* status, void* stream) {
  if (d && d->n_dur == 0) return FRNNT_ERR_DIMS;
  return fwd_bwd_impl(d, f, g, W_f, W_g, W_o, b_o, W_d, b_d, labels, T_len, U_len, nullptr, grad_loss, loss, df, dg,
                      dW_f, dW_g, dW_o, db_o, dW_d, db_d, workspace, workspace_bytes, status, stream);
}

extern "C" const char* frnnt_error_string(int code) {
  switch (code) {
    case FRNNT_OK: return "ok";
    case FRNNT_ERR_NULL: return "a required pointer is NULL";
    case FRNNT_ERR_DIMS:
      return "invalid dimensions (a size <= 0, blank outside [0,V), U+1 > 1024, a pruned / duration rule "
             "broken, or dims for another entry point)";
    case FRNNT_ERR_WORKSPACE: return "workspace smaller than frnnt_workspace_size";
    case FRNNT_ERR_UNSUPPORTED: return "unsupported dtype, mode or path";
    case FRNNT_ERR_CUDA: return "a CUDA launch failed";
    case FRNNT_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    default: break;
  }
  return "unknown frnnt code";
}

extern "C" const char* frnnt_version(void) { return "0.1.0"; }
