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
#include "frnnt_common.cuh"
#include "frnnt_internal.h"
#include "sm100.cuh"

namespace frnnt {

using namespace sm100;

namespace {

constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr int kMaxKB = 16;          // H <= 1024
constexpr int kDbSlots = 8;

enum JointMode { MODE_FWD = 0, MODE_FWD_STORE = 1, MODE_BWD_DZ = 2 };

struct JointParams {
  int T, U, H, V, blank, TB, UB;
  int KB;                 // H / 64
  int nV;                 // V / BN
  int stages;
  const float* F;         // [B*T][H] fp32
  const float* G;         // [B*(U+1)][H] fp32
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
  __nv_bfloat16* hbuf;    // FWD_STORE / BWD_DZ: h rows, same row indexing as zbuf
  float* db_part;         // BWD_DZ: [kDbSlots][V]
  int32_t* status;
};

struct RowInfo {
  bool valid;
  int b, t, u, Tb, Ub, y;
  size_t cell;            // padded lattice index
};

__device__ __forceinline__ RowInfo row_info(const JointParams& p, int4 tile, int r) {
  RowInfo ri;
  ri.b = tile.x;
  ri.t = tile.y + r / p.UB;
  ri.u = tile.z + r % p.UB;
  const Lengths l = lengths_of(p.T_len, p.U_len, ri.b, p.T, p.U);
  ri.Tb = l.Tb;
  ri.Ub = l.Ub;
  ri.valid = ri.t < l.Tb && ri.u <= l.Ub;
  ri.y = (ri.valid && ri.u < l.Ub) ? label_of(p.labels, ri.b, ri.u, p.U, p.V) : -1;
  ri.cell = ((size_t)ri.b * p.T + (ri.valid ? ri.t : 0)) * (p.U + 1) + (ri.valid ? ri.u : 0);
  return ri;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;

// Sum over the 32 lanes of v[j] for every j; lane l ends up with column l's
// total in v[0] (reduce-scatter by halving exchanges).
__device__ __forceinline__ float warp_column_sums(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int j = 0; j < k; ++j) {
      const float send = upper ? v[j] : v[j + k];
      const float keep = upper ? v[j + k] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, k);
    }
  }
  return v[0];
}

template <int BN, int MODE>
__global__ void __launch_bounds__(kThreads, 1) joint_tc_kernel(const __grid_constant__ CUtensorMap tmW, JointParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int STAGE_BYTES = BN * 128;
  uint8_t* hs = smem;                                   // KB x 16 KB
  uint8_t* ring = smem + p.KB * 16384;                  // stages x STAGE_BYTES
  uint64_t* full = (uint64_t*)(ring + p.stages * STAGE_BYTES);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* hfull = tempty + 2;
  uint64_t* hempty = hfull + kMaxKB;
  uint32_t* tmem_base_p = (uint32_t*)(hempty + kMaxKB);
  volatile int* abort_flag = (volatile int*)(tmem_base_p + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = min(p.tile_end, *p.ntiles);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    for (int i = 0; i < kMaxKB; ++i) {
      mbar_init(&hfull[i], 4);
      mbar_init(&hempty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_base_p, 2 * BN);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) tma_prefetch_desc(&tmW);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_p;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer: W_o tiles
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = p.tile_begin + blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        for (int n = 0; n < p.nV && ok; ++n) {
          for (int kb = 0; kb < p.KB; ++kb) {
            if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
            tma_load_2d(ring + s * STAGE_BYTES, &tmW, &full[s], kb * 64, n * BN);
            if (++s == p.stages) {
              s = 0;
              ph ^= 1;
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, false, false);
      int s = 0;
      uint32_t ph = 0;
      int acc_i = 0;
      uint32_t hph = 0;
      bool ok = true;
      const uint32_t hs_addr = smem_u32(hs);
      for (int tile = p.tile_begin + blockIdx.x; tile < ntiles && ok; tile += gridDim.x, hph ^= 1) {
        for (int n = 0; n < p.nV && ok; ++n, ++acc_i) {
          const int a = acc_i & 1;
          const uint32_t aph = (acc_i >> 1) & 1;
          if (!mbar_wait(&tempty[a], aph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tbase + a * BN;
          for (int kb = 0; kb < p.KB; ++kb) {
            if (n == 0 && !mbar_wait(&hfull[kb], hph, abort_flag)) {
              ok = false;
              break;
            }
            if (!mbar_wait(&full[s], ph, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = hs_addr + kb * 16384;
            const uint32_t sb = smem_u32(ring + s * STAGE_BYTES);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16_ss(dt, sdesc_sw128(sa + k * 32, 16, 1024), sdesc_sw128(sb + k * 32, 16, 1024), idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
            mma_commit(&empty[s]);
            if (n == p.nV - 1) mma_commit(&hempty[kb]);   // h block kb is free once these MMAs finish
            if (++s == p.stages) {
              s = 0;
              ph ^= 1;
            }
          }
          if (ok) mma_commit(&tfull[a]);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ h generation + epilogue (warps 0-3)
    const int tid = threadIdx.x;            // 0..127
    const int r = warp * 32 + lane;         // tile row owned in the epilogue
    const int H = p.H, V = p.V;
    const int Up1 = p.U + 1;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int acc_i = 0;
    uint32_t hph = 0;
    for (int tile = p.tile_begin + blockIdx.x; tile < ntiles; tile += gridDim.x, hph ^= 1) {
      const int4 td = p.tiles[tile];
      const size_t row_base = (MODE == MODE_BWD_DZ) ? (size_t)(tile - p.tile_begin) * 128 : (size_t)tile * 128;
      // rows this thread generates: (tid >> 3) + 16 i, i = 0..7; -1 marks a cell outside the lattice
      int frow[8], grow[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const RowInfo gi = row_info(p, td, (tid >> 3) + 16 * i);
        frow[i] = gi.valid ? gi.b * p.T + gi.t : -1;
        grow[i] = gi.b * Up1 + gi.u;
      }
      const int c8 = tid & 7;
      // ---- generate h, one 64-wide K block at a time
      for (int kb = 0; kb < p.KB; ++kb) {
        if (!mbar_wait(&hempty[kb], hph ^ 1, abort_flag)) break;
        uint8_t* blk = hs + kb * 16384;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int row = (tid >> 3) + 16 * i;
          uint4 packed = make_uint4(0, 0, 0, 0);
          if (frow[i] >= 0) {
            const float* Fr = p.F + (size_t)frow[i] * H + kb * 64 + c8 * 8;
            const float* Gr = p.G + (size_t)grow[i] * H + kb * 64 + c8 * 8;
            const float4 f0 = __ldg((const float4*)Fr), f1 = __ldg((const float4*)Fr + 1);
            const float4 g0 = __ldg((const float4*)Gr), g1 = __ldg((const float4*)Gr + 1);
            packed.x = pack_bf16x2(tanh_approx(f0.x + g0.x), tanh_approx(f0.y + g0.y));
            packed.y = pack_bf16x2(tanh_approx(f0.z + g0.z), tanh_approx(f0.w + g0.w));
            packed.z = pack_bf16x2(tanh_approx(f1.x + g1.x), tanh_approx(f1.y + g1.y));
            packed.w = pack_bf16x2(tanh_approx(f1.z + g1.z), tanh_approx(f1.w + g1.w));
          }
          *(uint4*)(blk + sw128_offset(row, c8 * 8)) = packed;
          if (MODE != MODE_FWD)
            *(uint4*)(p.hbuf + (row_base + row) * H + kb * 64 + c8 * 8) = packed;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&hfull[kb]);
      }
      if (*abort_flag) break;

      // ---- per-row state
      const RowInfo ri = row_info(p, td, r);
      float m = -INFINITY, ssum = 0.f, zb = 0.f, zy = 0.f;
      float lse = 0.f, bpost = 0.f, lpost = 0.f, occ = 0.f, w = 0.f;
      if (MODE == MODE_BWD_DZ && ri.valid) {
        const size_t c = ri.cell;
        const float logp = p.L.beta[(size_t)ri.b * p.T * Up1];
        const float al = p.L.alpha[c];
        float beta_t1;
        if (ri.t + 1 < ri.Tb) beta_t1 = p.L.beta[c + Up1];
        else beta_t1 = (ri.u == ri.Ub) ? 0.f : -INFINITY;
        lse = p.L.lse[c];
        bpost = __expf(al + p.L.blank_lp[c] + beta_t1 - logp);
        lpost = ri.u < ri.Ub ? __expf(al + p.L.label_lp[c] + p.L.beta[c + 1] - logp) : 0.f;
        occ = bpost + lpost;
        w = p.grad_loss ? p.grad_loss[ri.b] : 1.f;
      }

      // ---- epilogue over the V tiles
      for (int n = 0; n < p.nV; ++n, ++acc_i) {
        const int a = acc_i & 1;
        const uint32_t aph = (acc_i >> 1) & 1;
        if (!mbar_wait(&tfull[a], aph, abort_flag)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(tbase + lane_base + a * BN + c * 32, rr);
          tmem_wait_ld();
          const int col0 = n * BN + c * 32;
          float v[32];
          const uint4* bp = (const uint4*)(p.b_o + col0);
#pragma unroll
          for (int j8 = 0; j8 < 4; ++j8) {
            const uint4 bw = __ldg(bp + j8);
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bb[q]));
              v[8 * j8 + 2 * q] = __uint_as_float(rr[8 * j8 + 2 * q]) + bf.x;
              v[8 * j8 + 2 * q + 1] = __uint_as_float(rr[8 * j8 + 2 * q + 1]) + bf.y;
            }
          }
          if (MODE != MODE_BWD_DZ) {
            float cm = v[0];
#pragma unroll
            for (int j = 1; j < 32; ++j) cm = fmaxf(cm, v[j]);
            const float mn = fmaxf(m, cm);
            float acc = ssum * ex2((m - mn) * kLog2e);
            const float mk = mn * kLog2e;
#pragma unroll
            for (int j = 0; j < 32; ++j) acc += ex2(fmaf(v[j], kLog2e, -mk));
            ssum = acc;
            m = mn;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (col0 + j == p.blank) zb = v[j];
              if (col0 + j == ri.y) zy = v[j];
            }
            if (MODE == MODE_FWD_STORE) {
              uint4* dst = (uint4*)(p.zbuf + (row_base + r) * V + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                    pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                    pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
            }
          } else {
            const float lk = lse * kLog2e;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float d = occ * ex2(fmaf(v[j], kLog2e, -lk));
              if (col0 + j == p.blank) d -= bpost;
              if (col0 + j == ri.y) d -= lpost;
              v[j] = ri.valid ? d * w : 0.f;
            }
            uint4* dst = (uint4*)(p.zbuf + (row_base + r) * V + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                  pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
            const float colsum = warp_column_sums(v);
            atomicAdd(p.db_part + (size_t)(blockIdx.x % kDbSlots) * V + col0 + lane, colsum);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
      }
      if (*abort_flag) break;
      if (MODE != MODE_BWD_DZ && ri.valid) {
        const float l = m + __logf(ssum);
        p.L.lse[ri.cell] = l;
        p.L.blank_lp[ri.cell] = zb - l;
        p.L.label_lp[ri.cell] = ri.u < ri.Ub ? zy - l : -INFINITY;
      }
    }
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, 2 * BN);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, FRNNT_STATUS_TIMEOUT);
}

// ------------------------------------------------------------------ tile list
// Tiles of utterance b: ceil(T_len/TB) x ceil((U_len+1)/UB) blocks, u-blocks fastest.
__global__ void tiles_kernel(int B, int T, int U, int TB, int UB, const int32_t* __restrict__ T_len,
                             const int32_t* __restrict__ U_len, int4* __restrict__ tiles, int* __restrict__ ntiles) {
  __shared__ int offs[1025];
  __shared__ int counts[1024];
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const Lengths l = lengths_of(T_len, U_len, b, T, U);
    counts[b] = ((l.Tb + TB - 1) / TB) * ((l.Ub + 1 + UB - 1) / UB);
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
    const int nu = (l.Ub + 1 + UB - 1) / UB;
    for (int i = threadIdx.x; i < counts[b]; i += blockDim.x) {
      const int it = i / nu, iu = i % nu;
      tiles[offs[b] + i] = make_int4(b, it * TB, iu * UB, 0);
    }
  }
}

// ------------------------------------------------------------------ untiled backward: dz from stored z
__global__ void dz_from_z_kernel(JointParams p) {
  // one warp per row; rows of tiles [tile_begin, ntiles)
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int V = p.V, Up1 = p.U + 1;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)max(0, ntiles - p.tile_begin) * 128;
  extern __shared__ float dbs[];   // [V] block partial sums
  for (int k = threadIdx.x; k < V; k += blockDim.x) dbs[k] = 0.f;
  __syncthreads();
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < nrows;
       row += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int tile = p.tile_begin + (int)(row >> 7);
    const RowInfo ri = row_info(p, p.tiles[tile], (int)(row & 127));
    __nv_bfloat16* zr = p.zbuf + (size_t)tile * 128 * V + (size_t)(row & 127) * V;
    if (!ri.valid) {
      for (int k = lane * 8; k < V; k += 256) *(uint4*)(zr + k) = make_uint4(0, 0, 0, 0);
      continue;
    }
    const size_t c = ri.cell;
    const float logp = p.L.beta[(size_t)ri.b * p.T * Up1];
    const float al = p.L.alpha[c];
    float beta_t1;
    if (ri.t + 1 < ri.Tb) beta_t1 = p.L.beta[c + Up1];
    else beta_t1 = (ri.u == ri.Ub) ? 0.f : -INFINITY;
    const float lse = p.L.lse[c];
    const float bpost = __expf(al + p.L.blank_lp[c] + beta_t1 - logp);
    const float lpost = ri.u < ri.Ub ? __expf(al + p.L.label_lp[c] + p.L.beta[c + 1] - logp) : 0.f;
    const float occ = bpost + lpost;
    const float w = p.grad_loss ? p.grad_loss[ri.b] : 1.f;
    const float lk = lse * kLog2e;
    for (int k = lane * 8; k < V; k += 256) {
      uint4 zv = *(const uint4*)(zr + k);
      uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[q]));
        float d0 = occ * ex2(fmaf(zf.x, kLog2e, -lk));
        float d1 = occ * ex2(fmaf(zf.y, kLog2e, -lk));
        const int k0 = k + 2 * q;
        if (k0 == p.blank) d0 -= bpost;
        if (k0 + 1 == p.blank) d1 -= bpost;
        if (k0 == ri.y) d0 -= lpost;
        if (k0 + 1 == ri.y) d1 -= lpost;
        d0 *= w;
        d1 *= w;
        atomicAdd(&dbs[k0], d0);
        atomicAdd(&dbs[k0 + 1], d1);
        o[q] = pack_bf16x2(d0, d1);
      }
      *(uint4*)(zr + k) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < V; k += blockDim.x)
    atomicAdd(p.db_part + (size_t)(blockIdx.x % kDbSlots) * V + k, dbs[k]);
}

// ------------------------------------------------------------------ dtanh'd hidden gradient -> dF, dG
// dpre rows of the tiles in [tile_begin, ntiles) (bf16, rows (tile - row_tile0) * 128 + r):
// dF[b, t] += sum over the tile's u of dpre, dG[b, u] += sum over the tile's t.
__global__ void seg_reduce_kernel(JointParams p, const __nv_bfloat16* __restrict__ dpre, int row_tile0, float* dF,
                                  float* dG) {
  const int ntiles = min(p.tile_end, *p.ntiles);
  const int tile = p.tile_begin + blockIdx.x;
  if (tile >= ntiles) return;
  const int4 td = p.tiles[tile];
  const int H = p.H, TB = p.TB, UB = p.UB, Up1 = p.U + 1;
  const Lengths l = lengths_of(p.T_len, p.U_len, td.x, p.T, p.U);
  const __nv_bfloat16* base = dpre + (size_t)(tile - row_tile0) * 128 * H;
  // each thread owns 8 consecutive columns; dF rows first, then dG rows
  for (int c8 = threadIdx.x; c8 * 8 < H; c8 += blockDim.x) {
    for (int tl = 0; tl < TB; ++tl) {
      const int t = td.y + tl;
      if (t >= l.Tb) break;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int ul = 0; ul < UB; ++ul) {
        if (td.z + ul > l.Ub) break;
        const uint4 v = *(const uint4*)(base + (size_t)(tl * UB + ul) * H + c8 * 8);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[q]));
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      }
      float* dst = dF + ((size_t)td.x * p.T + t) * H + c8 * 8;
      red_add_v4(dst, acc[0], acc[1], acc[2], acc[3]);
      red_add_v4(dst + 4, acc[4], acc[5], acc[6], acc[7]);
    }
    for (int ul = 0; ul < UB; ++ul) {
      const int u = td.z + ul;
      if (u > l.Ub) break;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int tl = 0; tl < TB; ++tl) {
        if (td.y + tl >= l.Tb) break;
        const uint4 v = *(const uint4*)(base + (size_t)(tl * UB + ul) * H + c8 * 8);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[q]));
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      }
      float* dst = dG + ((size_t)td.x * Up1 + u) * H + c8 * 8;
      red_add_v4(dst, acc[0], acc[1], acc[2], acc[3]);
      red_add_v4(dst + 4, acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

__global__ void db_finalize_kernel(const float* __restrict__ db_part, int V, void* out, int to_bf16) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < V; k += gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int i = 0; i < kDbSlots; ++i) s += db_part[(size_t)i * V + k];
    if (to_bf16) ((__nv_bfloat16*)out)[k] = __float2bfloat16_rn(s);
    else ((float*)out)[k] = s;
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
constexpr int kBarBytes = 1024;

template <int BN>
int stages_for(int KB) {
  const int avail = kSmemLimit - 1024 - kBarBytes - KB * 16384;
  int st = avail / (BN * 128);
  return st > kMaxStages ? kMaxStages : st;
}

template <int BN, int MODE>
int launch_joint_t(const CUtensorMap& tm, JointParams p, cudaStream_t st) {
  p.stages = stages_for<BN>(p.KB);
  if (p.stages < 2) return FRNNT_ERR_UNSUPPORTED;
  const int smem = 1024 + p.KB * 16384 + p.stages * BN * 128 + kBarBytes;
  auto kern = joint_tc_kernel<BN, MODE>;
  static int attr_set = 0;
  if (attr_set < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
      return FRNNT_ERR_CUDA;
    attr_set = kSmemLimit;
  }
  kern<<<sms(), kThreads, smem, st>>>(tm, p);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FRNNT_OK : FRNNT_ERR_CUDA;
}

}  // namespace

// ------------------------------------------------------------------ host entry points
bool joint_tc_supported(int H, int V) {
  if (H % 64 || H > 1024 || V % 128) return false;
  const int KB = H / 64;
  return (V % 256 == 0) ? stages_for<256>(KB) >= 2 : stages_for<128>(KB) >= 2;
}

void tile_shape(int U, int* TB, int* UB) {
  // label positions per tile: a power of two near U+1 so ragged u-blocks waste little
  const int Up1 = U + 1;
  int ub = 16;
  if (Up1 <= 8) ub = 8;
  else if (Up1 <= 16) ub = 16;
  else if (Up1 <= 24) ub = 8;
  *UB = ub;
  *TB = 128 / ub;
}

long long max_tiles(const Shape& s, int TB, int UB) {
  return (long long)s.B * ((s.T + TB - 1) / TB) * ((s.Up1 + UB - 1) / UB);
}

void launch_tiles(const Shape& s, int TB, int UB, const int32_t* T_len, const int32_t* U_len, int4* tiles, int* ntiles,
                  cudaStream_t st) {
  tiles_kernel<<<1, 1024, 0, st>>>(s.B, s.T, s.U, TB, UB, T_len, U_len, tiles, ntiles);
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
  p.F = j.F;
  p.G = j.G;
  p.b_o = (const __nv_bfloat16*)j.b_o;
  p.labels = j.labels;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.grad_loss = j.grad_loss;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  p.L = j.L;
  p.zbuf = (__nv_bfloat16*)j.zbuf;
  p.hbuf = (__nv_bfloat16*)j.hbuf;
  p.db_part = j.db_part;
  p.status = j.status;
  const int BN = (p.V % 256 == 0) ? 256 : 128;
  p.nV = p.V / BN;
  CUtensorMap tm;
  if (!make_tmap_bf16_2d(&tm, j.W_o, p.H, p.V, p.H, 64, BN)) return FRNNT_ERR_CUDA;
  const int mode = j.mode;
  if (BN == 256) {
    if (mode == MODE_FWD) return launch_joint_t<256, MODE_FWD>(tm, p, st);
    if (mode == MODE_FWD_STORE) return launch_joint_t<256, MODE_FWD_STORE>(tm, p, st);
    return launch_joint_t<256, MODE_BWD_DZ>(tm, p, st);
  }
  if (mode == MODE_FWD) return launch_joint_t<128, MODE_FWD>(tm, p, st);
  if (mode == MODE_FWD_STORE) return launch_joint_t<128, MODE_FWD_STORE>(tm, p, st);
  return launch_joint_t<128, MODE_BWD_DZ>(tm, p, st);
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
  p.L = j.L;
  p.zbuf = (__nv_bfloat16*)j.zbuf;
  p.db_part = j.db_part;
  dz_from_z_kernel<<<sms() * 4, 256, (size_t)p.V * sizeof(float), st>>>(p);
  note_launch();
}

void launch_seg_reduce(const JointLaunch& j, const void* dpre, int row_tile0, float* dF, float* dG, cudaStream_t st) {
  JointParams p{};
  p.T = j.s.T;
  p.U = j.s.U;
  p.H = j.s.H;
  p.TB = j.TB;
  p.UB = j.UB;
  p.T_len = j.T_len;
  p.U_len = j.U_len;
  p.tiles = j.tiles;
  p.ntiles = j.ntiles;
  p.tile_begin = j.tile_begin;
  p.tile_end = j.tile_end;
  const int n = j.tile_end - j.tile_begin;
  if (n <= 0) return;
  int threads = (p.H / 8 + 31) / 32 * 32;
  if (threads > 128) threads = 128;
  seg_reduce_kernel<<<n, threads, 0, st>>>(p, (const __nv_bfloat16*)dpre, row_tile0, dF, dG);
  note_launch();
}

void launch_db_finalize(const float* db_part, int V, void* out, bool to_bf16, cudaStream_t st) {
  db_finalize_kernel<<<(V + 255) / 256, 256, 0, st>>>(db_part, V, out, to_bf16);
  note_launch();
}

}  // namespace frnnt
