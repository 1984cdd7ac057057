// Fused joint network on the tensor cores (tcgen05 / TMEM / TMA), bf16.
//
// A work tile is 128 lattice cells of one utterance: a TB x UB block of
// frames x label positions (TB * UB = 128).  For a tile the kernel
//   1. generates the hidden tile h = tanh(F[t] + G[u]) (128 x H, bf16) straight
//      into shared memory in the MMA's 128-byte-swizzled K-major layout, one
//      64-wide K block at a time, signalling each block to the MMA as soon as
//      it is written ("Transformer Transducer", abstract: the two encoders'
//      activations combined by a feed-forward layer for every frame / label
//      history pair);
//   2. streams W_o through a TMA ring and runs S = h W_o^T over the full
//      vocabulary in V tiles of BN columns, accumulating in TMEM (two BN-column
//      buffers, so the epilogue of one V tile overlaps the MMAs of the next);
//   3. epilogue, per cell (one TMEM lane per thread):
//        FWD      online log-sum-exp over the V tiles, plus the blank and label
//                 logits -> lse, blank_lp, label_lp (fp32) for the lattice;
//                 optionally also stores z (bf16) and h (bf16) for the untiled
//                 backward;
//        BWD_DZ   recomputes S and forms the logit gradient
//                 dz = w (occ softmax - bpost e_blank - lpost e_label) in
//                 registers, stores it (bf16) with h (bf16) into the chunk
//                 buffers that the dW_o and d_hidden GEMMs read, and reduces
//                 the per-column sums for db_o.
// ("Flash RNN-T", abstract: joint and loss with tiled recomputation over the
// alignment space and vocabulary.)
//
// Roles: warps 0-3 generate h and run the epilogue (warp w owns TMEM lanes
// 32w..32w+31 = tile rows), warp 4 issues TMA loads of W_o, warp 5 issues the
// MMAs.  Persistent: one CTA per SM walks the tile list.
#include <algorithm>

#include "frnnt_common.cuh"
#include "frnnt_internal.h"
#include "sm100.cuh"

namespace frnnt {

using namespace sm100;

void tile_shape(int T, int U, int* TB, int* UB);

namespace {

// warps 0-7 epilogue (two per TMEM lane quadrant, each half of a V tile's
// columns), warp 8 TMA, warp 9 MMA, warps 10-17 h generators (two per quadrant,
// each half of every K block)
constexpr int kThreads = 576;
constexpr int kEpiWarps = 8, kGenWarps = 8;
constexpr int kTmaWarp = 8, kMmaWarp = 9, kGen0 = 10;
constexpr int BN = 128;             // V tile (MMA N)
constexpr int kStageBytes = BN * 128;
constexpr int kMaxStages = 16;
constexpr int kMaxKB = 16;          // H <= 1024
constexpr int kTmemKB = 8;          // the first 8 K blocks (512 columns of h) live in TMEM
constexpr int kHCol = 256;          // TMEM columns: [0,128) and [128,256) accumulators, [256,512) h

// Shared memory of the staged F / G rows: TB + UB rows of 2H + 16 bytes, 1 KB aligned.
__host__ __device__ constexpr int fg_bytes(int TB, int UB, int H) { return (((TB + UB) * (2 * H + 16)) + 1023) & ~1023; }

enum JointMode { MODE_FWD = 0, MODE_FWD_STORE = 1, MODE_BWD_DZ = 2 };

struct JointParams {
  int T, U, H, V, blank, TB, UB;
  int KB;                 // H / 64
  int nV;                 // V / BN
  int stages;
  int ks;                 // 64-wide K blocks per h group (one generator signal; 1 or 2)
  int kr;                 // 64-wide K blocks per W_o ring stage (>= ks; one TMA / MMA hand-off)
  const __nv_bfloat16* F;   // [B*T][H] bf16
  const __nv_bfloat16* G;   // [B*(U+1)][H] bf16
  const __nv_bfloat16* b_o;
  const int32_t* labels;
  const int32_t* T_len;
  const int32_t* U_len;
  const float* grad_loss;
  const int4* tiles;      // (b, t0, u0, -)
  const int* ntiles;
  int tile_begin, tile_end;   // this launch's tile range (clamped by *ntiles)
  Lattice L;
  __nv_bfloat16* zbuf;    // FWD_STORE: z [tile*128 + r][V]; BWD_DZ: dz [(tile-tile_begin)*128 + r][V]
  __nv_bfloat16* hbuf;    // FWD_STORE / BWD_DZ: h rows [.][HS], same row indexing as zbuf; column H holds 1
  int HS;                 // row stride of hbuf (hidden_stride(H))
  int srows;              // epilogue store-staging rows per warp (0: stores go straight from registers)
  float* db_part;         // dz_db_kernel: db_o accumulator [V] (column sums of dz), else unused
  // BWD_DZ: per-row scalars of this launch's tiles (row_params_kernel), row
  // (tile - tile_begin) * 128 + r: (lse log2 e, w bpost, w lpost, label or -2
  // for no cell), so the epilogue needs one independent load per tile row
  const float4* rp;
  int32_t* status;
  const int32_t* bounds;  // pruned lattice: [B][T] band starts; S = band width (0: whole lattice)
  int S;
  // columns of the joint's output weights and row stride of zbuf: V, or for the
  // token-and-duration transducer (n_dur > 0) V + 128, the last 128-column tile
  // holding the duration head (columns V .. V + n_dur - 1)
  int Vx;
  int n_dur;
  // FWD_STORE / BWD_DZ: the generators also store the h rows they build into
  // hbuf (rows as zbuf's), with the column block [1, 0, ...] (0 outside the
  // lattice) after column H, for the backward GEMMs
  int store_h;
  // 1: the tile's F and G rows are bulk-copied into shared memory one tile
  // ahead; 0 (when shared memory is better spent on the W_o ring): the
  // generators read them from global memory (L2-resident)
  int stage_fg;
};

struct RowInfo {
  bool valid;
  int b, t, u, j, Tb, Ub, y;
  size_t cell;            // lattice index: [b][t][u] (padded), or [b][t][j] on a pruned lattice
};

// Cell of tile row r: frame t0 + r / UB and label position u0 + r % UB, or on
// a pruned lattice band position j = r % UB of frame t, u = bounds[b,t] + j.
__device__ __forceinline__ RowInfo row_info(const JointParams& p, int4 tile, int r) {
  RowInfo ri;
  ri.b = tile.x;
  ri.t = tile.y + r / p.UB;
  const Lengths l = lengths_of(p.T_len, p.U_len, ri.b, p.T, p.U);
  ri.Tb = l.Tb;
  ri.Ub = l.Ub;
  if (p.S) {
    ri.j = r % p.UB;
    const int tc = min(ri.t, l.Tb - 1);
    ri.u = clampi(p.bounds[(size_t)ri.b * p.T + tc], 0, p.U) + ri.j;
    ri.valid = ri.t < l.Tb && ri.j < p.S && ri.u <= l.Ub;
    ri.cell = ((size_t)ri.b * p.T + (ri.valid ? ri.t : 0)) * p.S + (ri.valid ? ri.j : 0);
  } else {
    ri.u = tile.z + r % p.UB;
    ri.j = ri.u;
    ri.valid = ri.t < l.Tb && ri.u <= l.Ub;
    ri.cell = ((size_t)ri.b * p.T + (ri.valid ? ri.t : 0)) * (p.U + 1) + (ri.valid ? ri.u : 0);
  }
  ri.y = (ri.valid && ri.u < l.Ub) ? label_of(p.labels, ri.b, ri.u, p.U, p.V) : -1;
  return ri;
}

// Lattice indices around a valid cell: the utterance's (0, 0), (t+1, u) and
// (t, u+1) (-1 when not in the lattice), and whether it is (T_len-1, U_len).
__device__ __forceinline__ void lattice_neighbors(const JointParams& p, const RowInfo& ri, size_t& c0, long long& c_t1,
                                                  long long& c_u1, bool& last) {
  last = ri.t == ri.Tb - 1 && ri.u == ri.Ub;
  if (p.S) {
    c0 = (size_t)ri.b * p.T * p.S;
    c_t1 = -1;
    if (ri.t + 1 < ri.Tb) {
      const int jn = ri.u - clampi(p.bounds[(size_t)ri.b * p.T + ri.t + 1], 0, p.U);
      if (jn >= 0 && jn < p.S) c_t1 = (long long)(c0 + (size_t)(ri.t + 1) * p.S + jn);
    }
    c_u1 = (ri.j + 1 < p.S && ri.u < ri.Ub) ? (long long)ri.cell + 1 : -1;
  } else {
    const int Up1 = p.U + 1;
    c0 = (size_t)ri.b * p.T * Up1;
    c_t1 = ri.t + 1 < ri.Tb ? (long long)(ri.cell + Up1) : -1;
    c_u1 = ri.u < ri.Ub ? (long long)ri.cell + 1 : -1;
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t tanh_bf16x2(uint32_t x) {
  uint32_t y;
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hadd2(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

constexpr float kLog2e = 1.4426950408889634f;

// Store one row's 32 bf16 (64 bytes, this lane's row of the tile) straight
// from registers with two 256-bit stores: every store fills one 32-byte
// sector, so no shared-memory staging is needed to write whole sectors (the
// staging's shared-memory traffic competed with the W_o operand stream).
__device__ __forceinline__ void store_row64(__nv_bfloat16* dst, const uint32_t (&w)[16]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 16), "r"(w[8]), "r"(w[9]),
               "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
               : "memory");
}

// PAIR: the CTAs of a 2-CTA cluster each own a cell tile (h, epilogue, F/G
// staging) and stage half of every W_o tile; the leader issues M = 256
// cta_group::2 MMAs over both, halving the W_o traffic per CTA.  Generator and
// epilogue signals go to the leader's barriers (cluster-scope release/acquire);
// the leader's commits reach both CTAs.
template <int MODE, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1) joint_tc_kernel(const __grid_constant__ CUtensorMap tmW, JointParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int KB_hi = p.KB > kTmemKB ? p.KB - kTmemKB : 0;
  uint8_t* hhi = smem;                                            // K blocks >= kTmemKB of h, 16 KB each
  uint8_t* ring = hhi + KB_hi * 16384;                            // stages x ks K blocks of W_o
  const int fg_stride = 2 * p.H + 16;                             // padded bf16 row (bank spread)
  constexpr int KBB = PAIR ? kStageBytes / 2 : kStageBytes;      // this CTA's rows of one K block of a W_o tile
  const int STAGE = p.kr * KBB;
  const int ngrp = (p.KB + p.ks - 1) / p.ks;                      // h groups of ks K blocks
  const int nst = (p.KB + p.kr - 1) / p.kr;                       // ring stages per V tile
  uint8_t* fgs = ring + p.stages * STAGE;                         // TB F rows then UB G rows of this tile
  __nv_bfloat16* bias_s = (__nv_bfloat16*)(fgs + (p.stage_fg ? fg_bytes(p.TB, p.UB, p.H) : 0));   // b_o (bf16)
  uint8_t* stage_s = (uint8_t*)(bias_s + ((p.Vx + 511) & ~511));  // per epilogue warp: srows x 80 B
  uint64_t* full = (uint64_t*)(stage_s + kEpiWarps * p.srows * 80);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* hfull = tempty + 2;
  uint64_t* hempty = hfull + kMaxKB;
  uint64_t* fg_full = hempty + kMaxKB;
  uint64_t* fg_empty = fg_full + 1;
  uint32_t* tmem_base_p = (uint32_t*)(fg_empty + 1);
  volatile int* abort_flag = (volatile int*)(tmem_base_p + 1);
  float* lse_x = (float*)(tmem_base_p + 4);       // [128][4] half-1 epilogue state for the combine

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  // iteration i of the persistent loop covers tile tile_begin + i (one CTA) or
  // tiles tile_begin + 2i and 2i + 1 (a pair; a missing odd tile is a dummy)
  const int slot = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int nslots = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  auto tile_of = [&](int i) { return p.tile_begin + (PAIR ? 2 * i + (int)rank : i); };
  // an empty tile range (a chunk past the device-built tile list): every CTA
  // of the grid sees the same count and leaves before any set-up or cluster
  // barrier, after waiting for the previous launch like every other launch
  if (min(p.tile_end, tile_count_early(p.ntiles)) <= p.tile_begin) {
    chain_wait();
    return;
  }
  // arrivals on barriers the (leader's) MMA thread waits for
  auto arrive_leader = [&](uint64_t* bar) {
    if (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(bar), 0));
    else mbar_arrive(bar);
  };
  auto commit_all = [&](uint64_t* bar) {
    if (PAIR) mma_commit_pair(bar, 0x3);
    else mma_commit(bar);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], PAIR ? 2 * kEpiWarps : kEpiWarps);
    }
    for (int i = 0; i < kMaxKB; ++i) {
      mbar_init(&hfull[i], PAIR ? 2 * kGenWarps : kGenWarps);
      mbar_init(&hempty[i], 1);
    }
    mbar_init(fg_full, 1);
    mbar_init(fg_empty, kGenWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    if (PAIR) {
      tmem_alloc_pair(tmem_base_p, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_base_p, 512);
      tmem_relinquish();
    }
  }
  if (warp == kTmaWarp && lane == 0) tma_prefetch_desc(&tmW);
  if (PAIR) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_p;
  // set-up done: from here on the previous launches' results are read
  chain_wait();
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int span = ntiles - p.tile_begin;
  const int niter = span <= 0 ? 0 : (PAIR ? (span + 1) / 2 : span);
  for (int k = threadIdx.x; k < p.Vx; k += blockDim.x) bias_s[k] = p.b_o[k];
  __syncthreads();

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer: W_o tiles
    // (the whole warp polls, one elected lane issues)
    {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = slot; it < niter && ok; it += nslots) {
        for (int n = 0; n < p.nV && ok; ++n) {
          for (int si = 0; si < nst; ++si) {
            if (!warp_wait(&empty[s], ph ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            const int kb0 = si * p.kr, nk = min(p.kr, p.KB - kb0);
            if (!elect_one()) {
              // other lanes: nothing to issue
            } else if (PAIR) {
              // both halves credit the leader's barrier, which expects both
              if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * nk * KBB);
              const uint32_t fl = mapa_shared(smem_u32(&full[s]), 0);
              for (int kk = 0; kk < nk; ++kk)
                tma_load_2d_pair(ring + s * STAGE + kk * KBB, &tmW, fl, (kb0 + kk) * 64, n * BN + (int)rank * (BN / 2));
            } else {
              mbar_arrive_expect_tx(&full[s], nk * KBB);
              for (int kk = 0; kk < nk; ++kk)
                tma_load_2d(ring + s * STAGE + kk * KBB, &tmW, &full[s], (kb0 + kk) * 64, n * BN);
            }
            __syncwarp();
            if (++s == p.stages) {
              s = 0;
              ph ^= 1;
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (the leader's warp; one elected lane issues)
    if (rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(PAIR ? 256 : 128, BN, false, false);
      int s = 0;
      uint32_t ph = 0;
      int acc_i = 0;
      uint32_t hph = 0;
      bool ok = true;
      const uint32_t hhi_addr = smem_u32(hhi);
      for (int it = slot; it < niter && ok; it += nslots, hph ^= 1) {
        for (int n = 0; n < p.nV && ok; ++n, ++acc_i) {
          const int a = acc_i & 1;
          const uint32_t aph = (acc_i >> 1) & 1;
          if (!(PAIR ? warp_wait_cluster(&tempty[a], aph ^ 1, abort_flag) : warp_wait(&tempty[a], aph ^ 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tbase + a * BN;
          int g_ready = 0;                  // h groups waited for in this tile (first V tile only)
          for (int si = 0; si < nst; ++si) {
            const int kb0 = si * p.kr, nk = min(p.kr, p.KB - kb0);
            if (n == 0) {
              // h groups the stage's K blocks belong to, written by the generators
              const int g_last = (kb0 + nk - 1) / p.ks;
              for (; g_ready <= g_last && ok; ++g_ready) {
                if (!(PAIR ? warp_wait_cluster(&hfull[g_ready], hph, abort_flag)
                           : warp_wait(&hfull[g_ready], hph, abort_flag)))
                  ok = false;
              }
              if (!ok) break;
              tc_fence_after();
            }
            // W_o stage landed (TMA completion is ordered by the mbarrier itself)
            if (!warp_wait(&full[s], ph, abort_flag)) {
              ok = false;
              break;
            }
            if (elect_one()) {
              for (int kk = 0; kk < nk; ++kk) {
                const int kb = kb0 + kk;
                const uint32_t sb = smem_u32(ring + s * STAGE + kk * KBB);
                if (kb < kTmemKB) {
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const uint32_t at = tbase + kHCol + kb * 32 + k * 8;
                    const uint64_t bd = sdesc_sw128(sb + k * 32, 16, 1024);
                    const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                    if (PAIR) mma_bf16_ts_pair(dt, at, bd, idesc, acc);
                    else mma_bf16_ts(dt, at, bd, idesc, acc);
                  }
                } else {
                  const uint32_t sa = hhi_addr + (kb - kTmemKB) * 16384;
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const uint64_t ad = sdesc_sw128(sa + k * 32, 16, 1024), bd = sdesc_sw128(sb + k * 32, 16, 1024);
                    if (PAIR) mma_bf16_ss_pair(dt, ad, bd, idesc, 1u);
                    else mma_bf16_ss(dt, ad, bd, idesc, 1u);
                  }
                }
              }
              commit_all(&empty[s]);
              if (n == p.nV - 1) {
                // an h group is free once the MMAs of its last K block finish
                for (int g = kb0 / p.ks; g < ngrp; ++g) {
                  const int g_end = min((g + 1) * p.ks, p.KB) - 1;
                  if (g_end >= kb0 + nk) break;
                  commit_all(&hempty[g]);
                }
              }
            }
            __syncwarp();
            if (++s == p.stages) {
              s = 0;
              ph ^= 1;
            }
          }
          if (ok && elect_one()) commit_all(&tfull[a]);
          __syncwarp();
        }
      }
    }
    __syncwarp();
  } else if (warp >= kGen0) {
    // ------------------------------------------------------------ h generators (warps 10-17)
    // The tile's TB rows of F and UB rows of G are bulk-copied into shared
    // memory (by warp kGen0, one tile ahead; without p.stage_fg every thread
    // reads its rows from global memory instead), then every thread builds its
    // row h[r, :] = tanh(F[t] + G[u]) 16 columns at a time (half of each
    // 64-wide K block per warp), into TMEM (first 512 columns of h) or the
    // swizzled shared-memory operand (the rest).
    const int q = warp & 3;                  // TMEM lane quadrant this warp may access
    const int half = (warp - kGen0) >> 2;    // which two of the four 16-column segments of each K block
    const int r = q * 32 + lane;             // tile row generated by this thread
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int H = p.H, Up1 = p.U + 1;
    uint32_t hph = 0;
    uint32_t fph = 0;
    // warp kGen0 only: wait until the generator warps are done with the buffer
    // (empty_parity 1 on the first call passes at once), then copy
    auto issue_fg = [&](int tile, uint32_t empty_parity) {
      const bool dummy = tile >= ntiles;
      const int4 td = dummy ? make_int4(0, p.T, 0, 0) : p.tiles[tile];
      // (a pruned lattice's G rows differ per frame: the generators read them from global memory)
      const int nF = dummy ? 0 : min(p.TB, p.T - td.y), nG = (dummy || p.S) ? 0 : min(p.UB, Up1 - td.z);
      if (!mbar_wait(fg_empty, empty_parity, abort_flag)) return false;
      if (lane == 0) mbar_arrive_expect_tx(fg_full, (uint32_t)(nF + nG) * H * 2);
      __syncwarp();
      if (lane < nF)
        bulk_load(fgs + lane * fg_stride, p.F + ((size_t)td.x * p.T + td.y + lane) * H, H * 2, fg_full);
      else if (lane >= 16 && lane - 16 < nG)
        bulk_load(fgs + (p.TB + lane - 16) * fg_stride, p.G + ((size_t)td.x * Up1 + td.z + lane - 16) * H, H * 2,
                  fg_full);
      return true;
    };
    bool ok = true;
    if (p.stage_fg && warp == kGen0 && slot < niter) ok = issue_fg(tile_of(slot), 1u);
    for (int it = slot; it < niter && ok; it += nslots, hph ^= 1, fph ^= 1) {
      const int tile = tile_of(it);
      // a dummy tile (the odd one out of a pair) has no valid row: its h is zero
      const int4 td = tile < ntiles ? p.tiles[tile] : make_int4(0, p.T, 0, 0);
      const RowInfo ri = row_info(p, td, r);
      // (global rows are read only for valid cells; the clamps keep the pointers in range regardless)
      const uint8_t* frow = p.stage_fg ? fgs + (r / p.UB) * fg_stride
                                       : (const uint8_t*)(p.F + ((size_t)ri.b * p.T + min(ri.t, p.T - 1)) * H);
      const uint8_t* grow = (p.S || !p.stage_fg) ? (const uint8_t*)(p.G + ((size_t)ri.b * Up1 + min(ri.u, p.U)) * H)
                                                 : fgs + (p.TB + r % p.UB) * fg_stride;
      if (p.stage_fg && !mbar_wait(fg_full, fph, abort_flag)) break;
      // h rows for the backward GEMMs (real tiles only; a pair's dummy tile has no rows)
      __nv_bfloat16* hrow = nullptr;
      if (MODE != MODE_FWD && p.store_h && tile < ntiles) {
        const size_t row0 = (MODE == MODE_BWD_DZ) ? (size_t)(tile - p.tile_begin) * 128 : (size_t)tile * 128;
        hrow = p.hbuf + (row0 + r) * p.HS;
        // bf16 1.0 in column H, zeros to H + 7; the dW_o GEMM reads the
        // columns past those as zeros (its operand's extent ends there)
        if (half == 0) *(uint4*)(hrow + H) = make_uint4(ri.valid ? 0x3F80u : 0u, 0u, 0u, 0u);
      }
      for (int g = 0; g < ngrp; ++g) {
        const int kb0 = g * p.ks, nk = min(p.ks, p.KB - kb0);
        // the whole group's values first (loads and MUFU work overlap the
        // wait for the MMAs to release the group), then the stores
        uint32_t pk[2][2][8];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int seg = (kb0 + kk) * 4 + 2 * half + j;
            if (kk < nk && ri.valid) {
              // h = tanh(F + G) in packed bf16 pairs (F, G already bf16; h is consumed as bf16)
              const uint4 f0 = *(const uint4*)(frow + seg * 32), f1 = *(const uint4*)(frow + seg * 32 + 16);
              const uint4 g0 = *(const uint4*)(grow + seg * 32), g1 = *(const uint4*)(grow + seg * 32 + 16);
              pk[kk][j][0] = tanh_bf16x2(add_bf16x2(f0.x, g0.x));
              pk[kk][j][1] = tanh_bf16x2(add_bf16x2(f0.y, g0.y));
              pk[kk][j][2] = tanh_bf16x2(add_bf16x2(f0.z, g0.z));
              pk[kk][j][3] = tanh_bf16x2(add_bf16x2(f0.w, g0.w));
              pk[kk][j][4] = tanh_bf16x2(add_bf16x2(f1.x, g1.x));
              pk[kk][j][5] = tanh_bf16x2(add_bf16x2(f1.y, g1.y));
              pk[kk][j][6] = tanh_bf16x2(add_bf16x2(f1.z, g1.z));
              pk[kk][j][7] = tanh_bf16x2(add_bf16x2(f1.w, g1.w));
            } else {
#pragma unroll
              for (int w = 0; w < 8; ++w) pk[kk][j][w] = 0u;
            }
            if (hrow && kk < nk) {
              // one 256-bit store: the row segment's whole 32-byte sector
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(hrow + seg * 16),
                           "r"(pk[kk][j][0]), "r"(pk[kk][j][1]), "r"(pk[kk][j][2]), "r"(pk[kk][j][3]),
                           "r"(pk[kk][j][4]), "r"(pk[kk][j][5]), "r"(pk[kk][j][6]), "r"(pk[kk][j][7])
                           : "memory");
            }
          }
        }
        if (!mbar_wait(&hempty[g], hph ^ 1, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          if (kk >= nk) break;
          const int kb = kb0 + kk;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int sub = 2 * half + j;
            if (kb < kTmemKB) {
              tmem_st8(tbase + lane_base + kHCol + kb * 32 + sub * 8, pk[kk][j]);
            } else {
              uint8_t* blk = hhi + (kb - kTmemKB) * 16384;
              *(uint4*)(blk + sw128_offset(r, sub * 16)) = make_uint4(pk[kk][j][0], pk[kk][j][1], pk[kk][j][2], pk[kk][j][3]);
              *(uint4*)(blk + sw128_offset(r, sub * 16 + 8)) =
                  make_uint4(pk[kk][j][4], pk[kk][j][5], pk[kk][j][6], pk[kk][j][7]);
            }
          }
        }
        // a group lies wholly in TMEM or wholly in shared memory
        if (kb0 < kTmemKB) {
          tmem_wait_st();
          tc_fence_before();
        } else {
          fence_proxy_async_smem();
        }
        __syncwarp();
        // TMEM groups are complete once tcgen05.wait::st returns (a relaxed
        // signal suffices); shared-memory groups are published with release
        if (lane == 0) {
          if (PAIR && kb0 < kTmemKB) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&hfull[g]), 0));
          else arrive_leader(&hfull[g]);
        }
      }
      if (!ok) break;
      if (p.stage_fg) {
        // this warp is done reading the tile's F/G rows
        __syncwarp();
        if (lane == 0) mbar_arrive(fg_empty);
        if (warp == kGen0 && it + nslots < niter) ok = issue_fg(tile_of(it + nslots), fph);
      }
      if (*abort_flag) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-7)
    const int q = warp & 3;                   // TMEM lane quadrant
    const int half = warp >> 2;               // columns [64 half, 64 half + 64) of each V tile
    const int r = q * 32 + lane;
    const int V = p.Vx;                       // row stride of zbuf
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int acc_i = 0;
    // BWD_DZ: the row's scalars, loaded one tile ahead
    auto load_rp = [&](int i) {
      const int tl = tile_of(i);
      return tl < ntiles ? p.rp[(size_t)(tl - p.tile_begin) * 128 + r] : make_float4(0.f, 0.f, 0.f, __int_as_float(-2));
    };
    float4 rp_next = make_float4(0.f, 0.f, 0.f, __int_as_float(-2));
    if (MODE == MODE_BWD_DZ && slot < niter) rp_next = load_rp(slot);
    for (int it = slot; it < niter; it += nslots) {
      const int tile = tile_of(it);
      const bool real = tile < ntiles;   // else the dummy of a pair: consume the accumulators, store nothing
      const size_t row_base = (MODE == MODE_BWD_DZ) ? (size_t)(tile - p.tile_begin) * 128 : (size_t)tile * 128;
      RowInfo ri;
      float m = -INFINITY, ssum = 0.f, zb = 0.f, zy = 0.f;
      float lk = 0.f, bpost = 0.f, lpost = 0.f, occ = 0.f;
      if (MODE == MODE_BWD_DZ) {
        const float4 rv = rp_next;
        if (it + nslots < niter) rp_next = load_rp(it + nslots);
        ri.y = __float_as_int(rv.w);
        ri.valid = ri.y != -2;
        lk = rv.x;
        bpost = rv.y;
        lpost = rv.z;
        occ = bpost + lpost;
      } else {
        ri = row_info(p, real ? p.tiles[tile] : make_int4(0, p.T, 0, 0), r);
      }
      bool ok = true;
      for (int n = 0; n < p.nV; ++n, ++acc_i) {
        const int a = acc_i & 1;
        const uint32_t aph = (acc_i >> 1) & 1;
        if (!mbar_wait(&tfull[a], aph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 2 * half; c < 2 * half + 2; ++c) {
          uint32_t buf[32];
          tmem_ld32(tbase + lane_base + a * BN + c * 32, buf);
          tmem_wait_ld();
          const int col0 = n * BN + c * 32;
          float v[32];
          const uint4* b8 = (const uint4*)(bias_s + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 bw = b8[j];
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bb[q]));
              v[8 * j + 2 * q] = __uint_as_float(buf[8 * j + 2 * q]) + bf.x;
              v[8 * j + 2 * q + 1] = __uint_as_float(buf[8 * j + 2 * q + 1]) + bf.y;
            }
          }
          if (MODE != MODE_BWD_DZ && p.n_dur > 0 && n == p.nV - 1) {
            // the duration head: its own log-softmax over columns 0 .. n_dur-1
            // of the last tile, not part of the label log-sum-exp, not stored
            if (c == 0 && half == 0 && real && ri.valid) {
              float md = v[0];
#pragma unroll
              for (int i = 1; i < FRNNT_MAX_DURATIONS; ++i)
                if (i < p.n_dur) md = fmaxf(md, v[i]);
              float sd = 0.f;
#pragma unroll
              for (int i = 0; i < FRNNT_MAX_DURATIONS; ++i)
                if (i < p.n_dur) sd += ex2((v[i] - md) * kLog2e);
              const float ld = md + __logf(sd);
#pragma unroll
              for (int i = 0; i < FRNNT_MAX_DURATIONS; ++i)
                if (i < p.n_dur) p.L.dur_lp[(size_t)i * p.L.plane + ri.cell] = v[i] - ld;
            }
          } else if (MODE != MODE_BWD_DZ) {
            float t0 = fmaxf(v[0], v[1]), t1 = fmaxf(v[2], v[3]);
#pragma unroll
            for (int j = 4; j < 32; j += 4) {
              t0 = fmaxf(t0, fmaxf(v[j], v[j + 1]));
              t1 = fmaxf(t1, fmaxf(v[j + 2], v[j + 3]));
            }
            const float mn = fmaxf(m, fmaxf(t0, t1));
            const float mk = mn * kLog2e;
            float s0 = ssum * ex2((m - mn) * kLog2e), s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              s0 += ex2(fmaf(v[j], kLog2e, -mk));
              s1 += ex2(fmaf(v[j + 1], kLog2e, -mk));
              s2 += ex2(fmaf(v[j + 2], kLog2e, -mk));
              s3 += ex2(fmaf(v[j + 3], kLog2e, -mk));
            }
            ssum = (s0 + s1) + (s2 + s3);
            m = mn;
            if (p.blank >= col0 && p.blank < col0 + 32) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j == p.blank) zb = v[j];
            }
            if (ri.y >= col0 && ri.y < col0 + 32) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j == ri.y) zy = v[j];
            }
            if (MODE == MODE_FWD_STORE && real) {
              uint32_t w[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
              store_row64(p.zbuf + (row_base + r) * V + col0, w);
            }
          } else if (real) {
            if (ri.valid) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = occ * ex2(fmaf(v[j], kLog2e, -lk));
              // the blank and label columns fall in one 32-column chunk each
              if (p.blank >= col0 && p.blank < col0 + 32) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (col0 + j == p.blank) v[j] -= bpost;
              }
              if (ri.y >= col0 && ri.y < col0 + 32) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (col0 + j == ri.y) v[j] -= lpost;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0.f;
            }
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
            store_row64(p.zbuf + (row_base + r) * V + col0, w);
          }
        }
        tc_fence_before();
        __syncwarp();
        // the accumulator is free (only TMEM was read: a relaxed signal suffices)
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&tempty[a]), 0));
          else mbar_arrive(&tempty[a]);
        }
      }
      if (!ok || *abort_flag) break;
      if (MODE != MODE_BWD_DZ) {
        // combine the two column halves of this row: half 1 hands its state to half 0
        if (half == 1) {
          lse_x[r * 4 + 0] = m;
          lse_x[r * 4 + 1] = ssum;
          lse_x[r * 4 + 2] = zb;
          lse_x[r * 4 + 3] = zy;
        }
        asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
        if (half == 0 && ri.valid) {
          const float m1 = lse_x[r * 4 + 0], s1 = lse_x[r * 4 + 1];
          const float mm = fmaxf(m, m1);
          const float st = ssum * ex2((m - mm) * kLog2e) + s1 * ex2((m1 - mm) * kLog2e);
          const float l = mm + __logf(st);
          const float zbb = zb + lse_x[r * 4 + 2], zyy = zy + lse_x[r * 4 + 3];
          p.L.lse[ri.cell] = l;
          p.L.blank_lp[ri.cell] = zbb - l;
          p.L.label_lp[ri.cell] = ri.u < ri.Ub ? zyy - l : -INFINITY;
        }
        asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
      }
    }
  }

  __syncthreads();
  if (PAIR) cluster_sync();   // no CTA leaves while its peer may still signal its barriers
  if (warp == kMmaWarp) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tbase, 512);
    else tmem_dealloc(tbase, 512);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, FRNNT_STATUS_TIMEOUT);
}

// ------------------------------------------------------------------ tile list
// Tiles of utterance b: ceil(T_len/TB) x ceil((U_len+1)/UB) blocks, u-blocks fastest
// (pruned: one tile per TB frames, its UB rows per frame being band positions);
// built by prologue_kernel below.

// ------------------------------------------------------------------ untiled backward: dz from stored z
// Token-and-duration transducer: the duration-head logit gradient of the cell
// behind row ri into the 128 bf16 columns at `out` (lane l writes columns
// 4l .. 4l+3):  dzd_i = w (occ P_dur(i) - exp(alpha - log P + q_i)) for
// i < n_dur, 0 past n_dur and for cells outside the lattice.
__device__ __forceinline__ void tdt_dzd_row(const JointParams& p, const RowInfo& ri, __nv_bfloat16* out, int lane) {
  float vals[4] = {0.f, 0.f, 0.f, 0.f};
  if (ri.valid && 4 * lane < p.n_dur) {
    size_t c0;
    long long c_t1, c_u1;
    bool last;
    lattice_neighbors(p, ri, c0, c_t1, c_u1, last);
    const size_t c = ri.cell;
    const float x = p.L.beta[c0], y = p.L.beta_l[c0];
    const float m = fmaxf(x, y);
    const float logp = m + __logf(__expf(x - m) + __expf(y - m));
    const float a = p.L.alpha[c] - logp;
    const float w = p.grad_loss ? p.grad_loss[ri.b] : 1.f;
    const float occ = __expf(a + p.L.beta[c]) + __expf(a + p.L.beta_l[c]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = 4 * lane + j;
      if (i < p.n_dur) {
        const size_t o = (size_t)i * p.L.plane + c;
        vals[j] = w * (occ * __expf(p.L.dur_lp[o]) - __expf(a + p.L.tdt_q[o]));
      }
    }
  }
  *(uint2*)(out + 4 * lane) = make_uint2(pack_bf16x2(vals[0], vals[1]), pack_bf16x2(vals[2], vals[3]));
}

// TDT: also write the duration columns (a separate instantiation, so the
// transducer's kernel keeps its register count and occupancy).
template <bool TDT>
__global__ void __launch_bounds__(256, 4) dz_from_z_kernel(JointParams p) {
  chain_wait();
  // one warp per row; rows of tiles [tile_begin, ntiles).  A row's z is read
  // in batches of four 16-byte chunks per lane, all loads of a batch issued
  // before any store (the row is rewritten in place).
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int V = p.V;
  const int ldz = p.Vx;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)max(0, ntiles - p.tile_begin) * 128;
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < nrows;
       row += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int tile = p.tile_begin + (int)(row >> 7);
    const RowInfo ri = row_info(p, p.tiles[tile], (int)(row & 127));
    __nv_bfloat16* zr = p.zbuf + (size_t)tile * 128 * ldz + (size_t)(row & 127) * ldz;
    if (TDT) tdt_dzd_row(p, ri, zr + V, lane);
    if (!ri.valid) {
      for (int k = lane * 8; k < V; k += 256) *(uint4*)(zr + k) = make_uint4(0, 0, 0, 0);
      continue;
    }
    const size_t c = ri.cell;
    const float lse = p.L.lse[c];
    const float w = p.grad_loss ? p.grad_loss[ri.b] : 1.f;
    float bpost, lpost;
    size_t c0;
    long long c_t1, c_u1;
    bool last;
    lattice_neighbors(p, ri, c0, c_t1, c_u1, last);
    edge_posteriors(p.L, c, c0, c_t1, c_u1, last, bpost, lpost);
    bpost *= w;
    lpost *= w;
    const float occ = bpost + lpost;
    const float lk = lse * kLog2e;
    for (int k0 = 0; k0 < V; k0 += 4 * 256) {
      uint4 zv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = k0 + i * 256 + lane * 8;
        if (k < V) zv[i] = *(const uint4*)(zr + k);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = k0 + i * 256 + lane * 8;
        if (k >= V) break;
        const uint32_t zw[4] = {zv[i].x, zv[i].y, zv[i].z, zv[i].w};
        float d[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[q]));
          d[2 * q] = occ * ex2(fmaf(zf.x, kLog2e, -lk));
          d[2 * q + 1] = occ * ex2(fmaf(zf.y, kLog2e, -lk));
        }
        // the blank and label columns fall in one 8-column group each
        if ((unsigned)(p.blank - k) < 8u) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (k + j == p.blank) d[j] -= bpost;
        }
        if ((unsigned)(ri.y - k) < 8u) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (k + j == ri.y) d[j] -= lpost;
        }
        *(uint4*)(zr + k) = make_uint4(pack_bf16x2(d[0], d[1]), pack_bf16x2(d[2], d[3]), pack_bf16x2(d[4], d[5]),
                                       pack_bf16x2(d[6], d[7]));
      }
    }
  }
}

// dz_from_z with the bias gradient: warps are split over the 1024-column ranges
// of the vocabulary, each warp owning one range (32 columns per lane) for all
// the rows it visits, so its column sums stay in registers; at the end every
// warp adds them to p.db_part.  Lets the dW_o GEMM run on N = H instead of a
// padded h with a ones column.  Rows: absolute tile rows (untiled).  TDT: the
// warps of range 0 also write the rows' duration columns.  The grid's warp
// count is a multiple of the number of ranges.
// Per-row scalars of the dz pass, computed once per row (the dz warps of
// several column ranges share them): {lse log2(e), w bpost, w lpost, label}
// with the label -2 for a row that is no lattice cell (-1: a cell without a
// label edge).
__global__ void row_params_kernel(JointParams p, float4* __restrict__ rp) {
  chain_wait();
  const int ntiles = min(p.tile_end, *p.ntiles);
  const long long nrows = (long long)max(0, ntiles - p.tile_begin) * 128;
  for (long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x; row < nrows;
       row += (long long)gridDim.x * blockDim.x) {
    const int tile = p.tile_begin + (int)(row >> 7);
    const RowInfo ri = row_info(p, p.tiles[tile], (int)(row & 127));
    float4 v = make_float4(0.f, 0.f, 0.f, __int_as_float(-2));
    if (ri.valid) {
      const float w = p.grad_loss ? p.grad_loss[ri.b] : 1.f;
      float bpost, lpost;
      size_t c0;
      long long c_t1, c_u1;
      bool last;
      lattice_neighbors(p, ri, c0, c_t1, c_u1, last);
      edge_posteriors(p.L, ri.cell, c0, c_t1, c_u1, last, bpost, lpost);
      v = make_float4(p.L.lse[ri.cell] * kLog2e, w * bpost, w * lpost, __int_as_float(ri.y));
    }
    rp[row] = v;
  }
}

template <bool TDT>
__global__ void __launch_bounds__(256, 3) dz_db_kernel(JointParams p, const float4* __restrict__ rp) {
  chain_wait();
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int V = p.V, ldz = p.Vx;
  const int lane = threadIdx.x & 31;
  const int ncr = (V + 1023) / 1024;
  const long long gw = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int cr = (int)(gw % ncr);
  const long long nw = (long long)gridDim.x * (blockDim.x >> 5) / ncr;
  const int k0 = cr * 1024;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const long long nrows = (long long)max(0, ntiles - p.tile_begin) * 128;
  // each row's scalars are fetched one iteration ahead, so the z loads of a
  // valid row (only those: rows that are no cell are just cleared) issue at once
  long long row = gw / ncr;
  float4 rv_next = row < nrows ? rp[row] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (; row < nrows; row += nw) {
    const float4 rv = rv_next;
    if (row + nw < nrows) rv_next = rp[row + nw];
    const int tile = p.tile_begin + (int)(row >> 7);
    __nv_bfloat16* zr = p.zbuf + (size_t)tile * 128 * ldz + (size_t)(row & 127) * ldz;
    if (TDT && cr == 0) tdt_dzd_row(p, row_info(p, p.tiles[tile], (int)(row & 127)), zr + V, lane);
    const int y = __float_as_int(rv.w);
    if (y == -2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = k0 + i * 256 + lane * 8;
        if (k < V) *(uint4*)(zr + k) = make_uint4(0, 0, 0, 0);
      }
      continue;
    }
    uint4 zv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = k0 + i * 256 + lane * 8;
      if (k < V) zv[i] = *(const uint4*)(zr + k);
    }
    const float lk = rv.x, bpost = rv.y, lpost = rv.z;
    const float occ = bpost + lpost;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = k0 + i * 256 + lane * 8;
      if (k >= V) break;
      const uint32_t zw[4] = {zv[i].x, zv[i].y, zv[i].z, zv[i].w};
      float d[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[q]));
        d[2 * q] = occ * ex2(fmaf(zf.x, kLog2e, -lk));
        d[2 * q + 1] = occ * ex2(fmaf(zf.y, kLog2e, -lk));
      }
      // the blank and label columns fall in one 8-column group each
      if ((unsigned)(p.blank - k) < 8u) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (k + j == p.blank) d[j] -= bpost;
      }
      if ((unsigned)(y - k) < 8u) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (k + j == y) d[j] -= lpost;
      }
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        o[q] = pack_bf16x2(d[2 * q], d[2 * q + 1]);
        // the bias gradient sums what the GEMMs read: the bf16-rounded dz
        const float2 r = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o[q]));
        acc[i][2 * q] += r.x;
        acc[i][2 * q + 1] += r.y;
      }
      *(uint4*)(zr + k) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = k0 + i * 256 + lane * 8;
    if (k < V) {
      red_add_v4(p.db_part + k, acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      red_add_v4(p.db_part + k + 4, acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
  }
}

// Tiled backward of the token-and-duration transducer: the duration columns of
// the chunk's dz rows (the label columns come from the joint kernel's dz pass).
__global__ void tdt_dzd_kernel(JointParams p) {
  chain_wait();
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)max(0, ntiles - p.tile_begin) * 128;
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < nrows;
       row += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int tile = p.tile_begin + (int)(row >> 7);
    const RowInfo ri = row_info(p, p.tiles[tile], (int)(row & 127));
    tdt_dzd_row(p, ri, p.zbuf + (size_t)row * p.Vx + p.V, lane);
  }
}

// W_x = [W_o; W_d; 0] (Vx rows of H) and b_x = [b_o; b_d; 0], bf16.
__global__ void tdt_weights_kernel(int V, int H, int n_dur, int Vx, const __nv_bfloat16* __restrict__ W_o,
                                   const __nv_bfloat16* __restrict__ b_o, const __nv_bfloat16* __restrict__ W_d,
                                   const __nv_bfloat16* __restrict__ b_d, __nv_bfloat16* __restrict__ W_x,
                                   __nv_bfloat16* __restrict__ b_x) {
  chain_wait();
  const int cpr = H / 8;                          // 16-byte chunks per row
  const long long n = (long long)Vx * cpr;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cpr), k = (int)(i % cpr) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < V) v = *(const uint4*)(W_o + (size_t)r * H + k);
    else if (r < V + n_dur) v = *(const uint4*)(W_d + (size_t)(r - V) * H + k);
    *(uint4*)(W_x + (size_t)r * H + k) = v;
  }
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < Vx; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)i;
    b_x[r] = r < V ? b_o[r] : (r < V + n_dur ? b_d[r - V] : __float2bfloat16_rn(0.f));
  }
}

// ------------------------------------------------------------------ hidden rows for the backward GEMMs
// h rows (bf16, stride HS = hidden_stride(H)) of tiles [tile_begin, ntiles) into hbuf rows
// (tile - row_tile0) * 128 + r: the same packed-bf16 tanh(F + G) as the joint
// kernel, plus the extra column block [1, 0, ..., 0] (0 for cells outside the
// lattice) whose dz-weighted sum is db_o.  One warp per row, coalesced.
__global__ void hidden_rows_kernel(JointParams p, int row_tile0) {
  chain_wait();
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int H = p.H, HS = p.HS, Up1 = p.U + 1;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)max(0, ntiles - p.tile_begin) * 128;
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < nrows;
       row += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int tile = p.tile_begin + (int)(row >> 7);
    const RowInfo ri = row_info(p, p.tiles[tile], (int)(row & 127));
    __nv_bfloat16* hr = p.hbuf + ((size_t)(tile - row_tile0) * 128 + (row & 127)) * HS;
    const __nv_bfloat16* Fr = p.F + ((size_t)ri.b * p.T + (ri.valid ? ri.t : 0)) * H;
    const __nv_bfloat16* Gr = p.G + ((size_t)ri.b * Up1 + (ri.valid ? ri.u : 0)) * H;
    // loads of up to four 16-byte chunks per lane issued before the stores
    for (int k0 = 0; k0 < H; k0 += 4 * 256) {
      uint4 f[4], g[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = k0 + i * 256 + lane * 8;
        if (k < H && ri.valid) {
          f[i] = *(const uint4*)(Fr + k);
          g[i] = *(const uint4*)(Gr + k);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = k0 + i * 256 + lane * 8;
        if (k >= H) break;
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (ri.valid) {
          o.x = tanh_bf16x2(add_bf16x2(f[i].x, g[i].x));
          o.y = tanh_bf16x2(add_bf16x2(f[i].y, g[i].y));
          o.z = tanh_bf16x2(add_bf16x2(f[i].z, g[i].z));
          o.w = tanh_bf16x2(add_bf16x2(f[i].w, g[i].w));
        }
        *(uint4*)(hr + k) = o;
      }
    }
    for (int k = H + lane * 8; k < HS; k += 256)
      *(uint4*)(hr + k) = make_uint4((k == H && ri.valid) ? 0x3F80u : 0u, 0u, 0u, 0u);
  }
}

// The same h rows, one block per cell tile (whole lattice): the tile's TB F rows
// and UB G rows are read once into shared memory (instead of once per row:
// each F row serves UB rows, each G row TB rows), then 8 warps write the
// tile's 128 rows, 16-byte stores.  Dynamic shared memory (TB + UB) H bf16.
__global__ void __launch_bounds__(256) hidden_tiles_kernel(JointParams p, int row_tile0) {
  chain_wait();
  extern __shared__ __align__(16) __nv_bfloat16 fg_s[];   // [TB][H] F rows, then [UB][H] G rows
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int H = p.H, HS = p.HS, Up1 = p.U + 1, TB = p.TB, UB = p.UB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cpr = H / 8;                                    // 16-byte chunks per row
  for (int tile = p.tile_begin + blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int4 td = p.tiles[tile];
    __syncthreads();                                        // the previous tile's rows are written
    for (int i = threadIdx.x; i < (TB + UB) * cpr; i += blockDim.x) {
      const int rr = i / cpr, k = (i % cpr) * 8;
      const __nv_bfloat16* src = rr < TB ? p.F + ((size_t)td.x * p.T + min(td.y + rr, p.T - 1)) * H
                                         : p.G + ((size_t)td.x * Up1 + min(td.z + rr - TB, p.U)) * H;
      *(uint4*)(fg_s + (size_t)rr * H + k) = __ldg((const uint4*)(src + k));
    }
    __syncthreads();
    for (int r = warp; r < 128; r += blockDim.x >> 5) {
      const RowInfo ri = row_info(p, td, r);
      __nv_bfloat16* hr = p.hbuf + ((size_t)(tile - row_tile0) * 128 + r) * HS;
      const __nv_bfloat16* Fr = fg_s + (size_t)(r / UB) * H;
      const __nv_bfloat16* Gr = fg_s + (size_t)(TB + r % UB) * H;
      for (int k = lane * 8; k < H; k += 256) {
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (ri.valid) {
          const uint4 f = *(const uint4*)(Fr + k), g = *(const uint4*)(Gr + k);
          o.x = tanh_bf16x2(add_bf16x2(f.x, g.x));
          o.y = tanh_bf16x2(add_bf16x2(f.y, g.y));
          o.z = tanh_bf16x2(add_bf16x2(f.z, g.z));
          o.w = tanh_bf16x2(add_bf16x2(f.w, g.w));
        }
        // streaming stores (evict first): the rows are read back only by the
        // later GEMMs, and should not push the concurrent DP's data out of L2
        __stcs((uint4*)(hr + k), o);
      }
      for (int k = H + lane * 8; k < HS; k += 256)
        __stcs((uint4*)(hr + k), make_uint4((k == H && ri.valid) ? 0x3F80u : 0u, 0u, 0u, 0u));
    }
  }
}

// dW_o [V][H] and db_o [V] (bf16, or fp32 when OUT_F32) out of the extended
// fp32 accumulator [V][HS] whose column H is the sum of dz over cells.
template <bool OUT_F32>
__global__ void wo_finalize_kernel(const float* __restrict__ acc, int V, int H, int HS, const float* __restrict__ db,
                                   void* __restrict__ dW_o, void* __restrict__ db_o) {
  chain_wait();
  const long long n = (long long)V * H;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long k = i / H, j = i % H;
    const float w = acc[k * HS + j];
    if (OUT_F32) ((float*)dW_o)[i] = w;
    else ((__nv_bfloat16*)dW_o)[i] = __float2bfloat16_rn(w);
    if (j == 0) {
      const float bias = db ? db[k] : acc[k * HS + H];
      if (OUT_F32) ((float*)db_o)[k] = bias;
      else ((__nv_bfloat16*)db_o)[k] = __float2bfloat16_rn(bias);
    }
  }
}

int sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

constexpr int kSmemLimit = 232448;   // max dynamic shared memory per block on sm_100
constexpr int kBarBytes = 3072;   // mbarriers + TMEM address + abort flag + 2 KB epilogue combine area

int smem_fixed(int KB, int V, int TB, int UB, int srows, bool stage_fg = true) {
  const int KB_hi = KB > kTmemKB ? KB - kTmemKB : 0;
  return 1024 + KB_hi * 16384 + (stage_fg ? fg_bytes(TB, UB, KB * 64) : 0) + ((V + 511) & ~511) * 2 +
         kEpiWarps * srows * 80 + kBarBytes;
}

// Staging rows: 32 when that still leaves at least 6 full W_o tiles of ring, else 8.
// (the epilogue stores straight from registers: no staging rows)
int staging_rows(int, int, int, int, bool = true) { return 0; }

// Ring stages of stage_bytes each (a full W_o tile, or half of one per CTA of a pair).
int stages_for(int KB, int V, int TB, int UB, int stage_bytes = kStageBytes, bool stage_fg = true) {
  int st = (kSmemLimit - smem_fixed(KB, V, TB, UB, staging_rows(KB, V, TB, UB, stage_fg), stage_fg)) / stage_bytes;
  return st > kMaxStages ? kMaxStages : st;
}

int g_joint_variant = -1;   // -1 automatic, 0 one CTA per tile, 1 CTA pairs

template <int MODE, bool PAIR>
int launch_joint_t(const CUtensorMap& tm, JointParams p, int ntiles_max, cudaStream_t st) {
  constexpr int kb_bytes = PAIR ? kStageBytes / 2 : kStageBytes;
  int stage_bytes = 0;
  auto plan = [&](bool fg) {
    p.stage_fg = fg ? 1 : 0;
    p.srows = staging_rows(p.KB, p.Vx, p.TB, p.UB, fg);
    // two K blocks per ring stage (half as many barrier polls in the MMA issuer)
    // while that still leaves at least three stages
    p.ks = stages_for(p.KB, p.Vx, p.TB, p.UB, 2 * kb_bytes, fg) >= 3 ? 2 : 1;
    // ring stages of up to 4 K blocks while two stages still fit: fewer
    // stage hand-offs per MMA (measured: 4 blocks beat 2 on medium and large,
    // most in the forward pass without z stores)
    p.kr = p.ks;
    for (int kr = 4; kr > p.ks; --kr)
      if (stages_for(p.KB, p.Vx, p.TB, p.UB, kr * kb_bytes, fg) >= 2) {
        p.kr = kr;
        break;
      }
    stage_bytes = p.kr * kb_bytes;
    p.stages = stages_for(p.KB, p.Vx, p.TB, p.UB, stage_bytes, fg);
  };
  // stage the F / G rows in shared memory unless that leaves the W_o ring
  // under 96 KB (large H: then the ring's depth matters more than the
  // generators' load latency, measured on H = 1024 vs 640)
  plan(true);
  if (p.stages * stage_bytes < 96 * 1024) plan(false);
  if (p.stages < 2) return FRNNT_ERR_UNSUPPORTED;
  const int smem = smem_fixed(p.KB, p.Vx, p.TB, p.UB, p.srows, p.stage_fg != 0) + p.stages * stage_bytes;
  auto kern = joint_tc_kernel<MODE, PAIR>;
  static bool attr_set[kDeviceSlots] = {};
  const int dev = current_device();
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
      return FRNNT_ERR_CUDA;
    attr_set[dev] = true;
  }
  if (!PAIR) {
    launch_k(kern, dim3(sms()), dim3(kThreads), smem, st, 1, tm, p);
  } else {
    // one cluster of two CTAs per pair of tiles; persistent, so no more
    // clusters than can be resident at once (an SM left without a partner in
    // its GPC stays idle)
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = 2;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    static int resident[kDeviceSlots] = {}, resident_smem[kDeviceSlots] = {};
    if (resident_smem[dev] != smem) {
      cfg.gridDim = dim3(sms(), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sms() / 2;
      }
      resident[dev] = n < sms() / 2 ? n : sms() / 2;
      resident_smem[dev] = smem;
    }
    const int pairs = (ntiles_max + 1) / 2;
    const int npairs = pairs < resident[dev] ? (pairs > 0 ? pairs : 1) : resident[dev];
    if (launch_k(kern, dim3(2 * npairs), dim3(kThreads), smem, st, 2, tm, p) != cudaSuccess) {
      note_launch();
      return FRNNT_ERR_CUDA;
    }
  }
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FRNNT_OK : FRNNT_ERR_CUDA;
}

}  // namespace

// ------------------------------------------------------------------ host entry points
bool joint_tc_supported(int H, int V, int T, int U, int S) {
  if (H % 64 || H > 1024 || V % 128) return false;
  Shape s{};
  s.T = T;
  s.U = U;
  s.S = S;
  int TB, UB;
  tile_shape_of(s, &TB, &UB);
  return stages_for(H / 64, V, TB, UB, kStageBytes, false) >= 2;
}

void tile_shape(int T, int U, int* TB, int* UB) {
  // label positions per tile.  Up to 16 positions fit one u-block (8 when
  // that is enough, with 16 frames); above that, the padding of the ragged
  // tiles at an utterance's edges grows as TB * (U_len+1) + UB * T_len, so
  // for lengths in proportion to T and U+1 eight positions by 16 frames pad
  // less than 16 by 8 whenever U+1 < T (both keep 24 F and G rows per tile)
  const int Up1 = U + 1;
  int ub;
  if (Up1 <= 8) ub = 8;
  else if (Up1 <= 16) ub = 16;
  else ub = Up1 < T ? 8 : 16;
  *UB = ub;
  *TB = 128 / ub;
}

void tile_shape_of(const Shape& s, int* TB, int* UB) {
  if (s.S > 0) {
    int sp = 4;                     // at most 32 frames per tile (their F rows are staged)
    while (sp < s.S) sp *= 2;
    *UB = sp;
    *TB = 128 / sp;
  } else {
    tile_shape(s.T, s.U, TB, UB);
  }
}

long long max_tiles(const Shape& s, int TB, int UB) {
  return (long long)s.B * ((s.T + TB - 1) / TB) * (s.S > 0 ? 1 : (s.Up1 + UB - 1) / UB);
}

// Block 0: the length / label validation and the tile list (a prefix sum of
// the per-utterance tile counts); the other blocks clear the accumulators.
__global__ void __launch_bounds__(1024) prologue_kernel(int B, int T, int U, int V, int blank, int TB, int UB,
                                                        int pruned, const int32_t* __restrict__ labels,
                                                        const int32_t* __restrict__ T_len,
                                                        const int32_t* __restrict__ U_len, int32_t* status,
                                                        int4* __restrict__ tiles, int* __restrict__ ntiles,
                                                        ZeroList z) {
  chain_wait();
  if (blockIdx.x > 0) {
    const long long stride = (long long)(gridDim.x - 1) * blockDim.x;
    const long long tid = (long long)(blockIdx.x - 1) * blockDim.x + threadIdx.x;
    for (int k = 0; k < z.count; ++k) {
      float4* p = (float4*)z.ptr[k];
      const long long n4 = z.n[k] / 4;
      for (long long i = tid; i < n4; i += stride) p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  int bits = validate_bits(B, T, U, V, blank, labels, T_len, U_len, threadIdx.x, blockDim.x);
  bits = __reduce_or_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0 && bits) atomicOr(status, bits);
  __shared__ int offs[1025];
  __shared__ int counts[1024];
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const Lengths l = lengths_of(T_len, U_len, b, T, U);
    counts[b] = ((l.Tb + TB - 1) / TB) * (pruned ? 1 : (l.Ub + 1 + UB - 1) / UB);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int b = 0; b < B; ++b) {
      offs[b] = acc;
      acc += counts[b];
    }
    offs[B] = acc;
    *ntiles = acc;
  }
  __syncthreads();
  for (int b = 0; b < B; ++b) {
    const Lengths l = lengths_of(T_len, U_len, b, T, U);
    const int nu = pruned ? 1 : (l.Ub + 1 + UB - 1) / UB;
    for (int i = threadIdx.x; i < counts[b]; i += blockDim.x) {
      const int it = i / nu, iu = i % nu;
      tiles[offs[b] + i] = make_int4(b, it * TB, iu * UB, 0);
    }
  }
}

void launch_prologue(const Shape& s, int TB, int UB, const int32_t* labels, const int32_t* T_len,
                     const int32_t* U_len, int32_t* status, int4* tiles, int* ntiles, const ZeroList& z,
                     cudaStream_t st) {
  long long total = 0;
  for (int k = 0; k < z.count; ++k) total += z.n[k];
  int zb = (int)((total / 4 + 1023) / 1024);
  if (zb > 2 * sms()) zb = 2 * sms();
  if (zb < 1) zb = 1;
  launch_k(prologue_kernel, dim3(1 + zb), dim3(1024), 0, st, 1, s.B, s.T, s.U, s.V, s.blank, TB, UB, s.S > 0 ? 1 : 0, labels, T_len,
                                           U_len, status, tiles, ntiles, z);
  note_launch();
}

int launch_joint_tc(const JointLaunch& j, cudaStream_t st) {
  JointParams p;
  p.T = j.s.T;
  p.U = j.s.U;
  p.H = j.s.H;
  p.V = j.s.V;
  p.blank = j.s.blank;
  p.TB = j.TB;
  p.UB = j.UB;
  p.KB = j.s.H / 64;
  p.F = (const __nv_bfloat16*)j.F;
  p.G = (const __nv_bfloat16*)j.G;
  p.b_o = (const __nv_bfloat16*)j.b_o;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.grad_loss = j.grad_loss;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.bounds = j.bounds;
  p.S = j.s.S;
  p.L = j.L;
  p.zbuf = (__nv_bfloat16*)j.zbuf;
  p.hbuf = (__nv_bfloat16*)j.hbuf;
  p.HS = hidden_stride(j.s.H);
  p.db_part = j.db_part;
  p.status = j.status;
  p.Vx = j.s.Vx;
  p.n_dur = j.s.n_dur;
  p.store_h = j.store_h;
  p.rp = j.row_params;
  if (j.mode == MODE_BWD_DZ && !p.rp) return FRNNT_ERR_CUDA;   // launch_row_params first
  // the backward dz pass covers the label tiles only (the duration head's
  // gradient comes from the stored duration log-probs)
  p.nV = (j.mode == MODE_BWD_DZ ? p.V : p.Vx) / BN;
  // upper bound of this launch's tile count (the exact count is on the device)
  const long long span = (long long)std::min<long long>(j.tile_end, max_tiles(j.s, j.TB, j.UB)) - j.tile_begin;
  const int ntiles_max = (int)std::max<long long>(0, span);
  // CTA pairs pay off when W_o is large (each CTA then streams half of it
  // through its shared memory, whose bandwidth bounds the one-CTA kernel); for
  // small W_o the coupling of the two CTAs' h generation costs more (measured:
  // pairs win from V H = 655k, medium, by 3-5 % in the forward and the
  // recompute pass, and by 25 % at 4.2M, large)
  const bool pair = g_joint_variant == 1 ||
                    (g_joint_variant < 0 && ntiles_max >= sms() && (long long)p.Vx * p.H >= (1LL << 19));
  CUtensorMap tm;
  // a pair CTA stages 64 of the BN rows of every W_o tile
  if (!make_tmap_bf16_2d(&tm, j.W_o, p.H, p.Vx, p.H, 64, pair ? BN / 2 : BN)) return FRNNT_ERR_CUDA;
  if (pair) {
    if (j.mode == MODE_FWD) return launch_joint_t<MODE_FWD, true>(tm, p, ntiles_max, st);
    if (j.mode == MODE_FWD_STORE) return launch_joint_t<MODE_FWD_STORE, true>(tm, p, ntiles_max, st);
    return launch_joint_t<MODE_BWD_DZ, true>(tm, p, ntiles_max, st);
  }
  if (j.mode == MODE_FWD) return launch_joint_t<MODE_FWD, false>(tm, p, ntiles_max, st);
  if (j.mode == MODE_FWD_STORE) return launch_joint_t<MODE_FWD_STORE, false>(tm, p, ntiles_max, st);
  return launch_joint_t<MODE_BWD_DZ, false>(tm, p, ntiles_max, st);
}

int set_joint_variant(int variant) {
  const int prev = g_joint_variant;
  g_joint_variant = variant < 0 ? -1 : (variant > 1 ? 1 : variant);
  return prev;
}

void launch_dz_from_z(const JointLaunch& j, cudaStream_t st) {
  JointParams p{};
  p.T = j.s.T;
  p.U = j.s.U;
  p.H = j.s.H;
  p.V = j.s.V;
  p.blank = j.s.blank;
  p.TB = j.TB;
  p.UB = j.UB;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.grad_loss = j.grad_loss;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.bounds = j.bounds;
  p.S = j.s.S;
  p.L = j.L;
  p.zbuf = (__nv_bfloat16*)j.zbuf;
  p.Vx = j.s.Vx;
  p.n_dur = j.s.n_dur;
  if (p.n_dur > 0) launch_k(dz_from_z_kernel<true>, dim3(sms() * 4), dim3(256), 0, st, 1, p);
  else launch_k(dz_from_z_kernel<false>, dim3(sms() * 4), dim3(256), 0, st, 1, p);
  note_launch();
}

void launch_dz_db(const JointLaunch& j, float* db_acc, float4* row_params, cudaStream_t st) {
  JointParams p{};
  p.T = j.s.T;
  p.U = j.s.U;
  p.H = j.s.H;
  p.V = j.s.V;
  p.blank = j.s.blank;
  p.TB = j.TB;
  p.UB = j.UB;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.grad_loss = j.grad_loss;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.bounds = j.bounds;
  p.S = j.s.S;
  p.L = j.L;
  p.zbuf = (__nv_bfloat16*)j.zbuf;
  p.Vx = j.s.Vx;
  p.n_dur = j.s.n_dur;
  p.db_part = db_acc;
  // 8 warps per block: the warp count sms * 3 * 8 is a multiple of the range count (1..4)
  const int ncr = (j.s.V + 1023) / 1024;
  int blocks = sms() * 3;
  blocks -= blocks % (ncr == 3 ? 3 : 1);
  launch_k(row_params_kernel, dim3(sms() * 8), dim3(256), 0, st, 1, p, row_params);
  note_launch();
  if (p.n_dur > 0) launch_k(dz_db_kernel<true>, dim3(blocks), dim3(256), 0, st, 1, p, row_params);
  else launch_k(dz_db_kernel<false>, dim3(blocks), dim3(256), 0, st, 1, p, row_params);
  note_launch();
}

bool dz_db_supported(int V, int H) { return V % 256 == 0 && V <= 4096 && H % 256 == 0; }

void launch_row_params(const JointLaunch& j, float4* row_params, cudaStream_t st) {
  JointParams p{};
  p.T = j.s.T;
  p.U = j.s.U;
  p.H = j.s.H;
  p.V = j.s.V;
  p.blank = j.s.blank;
  p.TB = j.TB;
  p.UB = j.UB;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.grad_loss = j.grad_loss;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.bounds = j.bounds;
  p.S = j.s.S;
  p.L = j.L;
  p.Vx = j.s.Vx;
  p.n_dur = j.s.n_dur;
  const long long rows = (long long)(j.tile_end - j.tile_begin) * 128;
  long long blocks = (rows + 255) / 256;
  if (blocks > sms() * 8) blocks = sms() * 8;
  if (blocks < 1) blocks = 1;
  launch_k(row_params_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 1, p, row_params);
  note_launch();
}

void launch_tdt_dzd(const JointLaunch& j, cudaStream_t st) {
  JointParams p{};
  p.T = j.s.T;
  p.U = j.s.U;
  p.V = j.s.V;
  p.TB = j.TB;
  p.UB = j.UB;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.grad_loss = j.grad_loss;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.bounds = j.bounds;
  p.S = j.s.S;
  p.L = j.L;
  p.zbuf = (__nv_bfloat16*)j.zbuf;
  p.Vx = j.s.Vx;
  p.n_dur = j.s.n_dur;
  launch_k(tdt_dzd_kernel, dim3(sms() * 4), dim3(256), 0, st, 1, p);
  note_launch();
}

void launch_tdt_weights(const Shape& s, const void* W_o, const void* b_o, const void* W_d, const void* b_d, void* W_x,
                        void* b_x, cudaStream_t st) {
  launch_k(tdt_weights_kernel, dim3(sms() * 2), dim3(256), 0, st, 1, s.V, s.H, s.n_dur, s.Vx, (const __nv_bfloat16*)W_o,
                                                (const __nv_bfloat16*)b_o, (const __nv_bfloat16*)W_d,
                                                (const __nv_bfloat16*)b_d, (__nv_bfloat16*)W_x, (__nv_bfloat16*)b_x);
  note_launch();
}

void launch_hidden_rows(const JointLaunch& j, int row_tile0, cudaStream_t st, int blocks_per_sm) {
  JointParams p{};
  p.T = j.s.T;
  p.U = j.s.U;
  p.H = j.s.H;
  p.V = j.s.V;
  p.TB = j.TB;
  p.UB = j.UB;
  p.HS = hidden_stride(j.s.H);
  p.F = (const __nv_bfloat16*)j.F;
  p.G = (const __nv_bfloat16*)j.G;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.bounds = j.bounds;
  p.S = j.s.S;
  p.hbuf = (__nv_bfloat16*)j.hbuf;
  if (j.s.S == 0) {
    // whole lattice: one block per cell tile, F and G rows read once per tile
    const int smem = (j.TB + j.UB) * j.s.H * 2;
    static int smem_set[kDeviceSlots] = {};
    const int dev = current_device();
    if (smem > 48 * 1024 && smem > smem_set[dev]) {
      cudaFuncSetAttribute(hidden_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      smem_set[dev] = smem;
    }
    // up to 6 resident blocks per SM (measured best beside the DP on medium),
    // fewer when their shared memory does not fit: one full wave
    int hb = (220 * 1024) / smem;
    hb = hb < 1 ? 1 : (hb > 6 ? 6 : hb);
    launch_k(hidden_tiles_kernel, dim3(sms() * hb), dim3(256), smem, st, 1, p, row_tile0);
  } else {
    launch_k(hidden_rows_kernel, dim3(sms() * blocks_per_sm), dim3(256), 0, st, 1, p, row_tile0);
  }
  note_launch();
}

void launch_wo_finalize(const float* acc, int V, int H, void* dW_o, void* db_o, cudaStream_t st, const float* db,
                        bool out_f32) {
  long long n = (long long)V * H;
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (out_f32)
    launch_k(wo_finalize_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, st, 1, acc, V, H, hidden_stride(H), db, dW_o, db_o);
  else
    launch_k(wo_finalize_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, st, 1, acc, V, H, hidden_stride(H), db, dW_o, db_o);
  note_launch();
}

}  // namespace frnnt
