// Persistent, warp-specialised bf16 GEMM on the 5th-generation tensor cores:
//   D[M,N] (fp32, TMEM) = A[M,K] * B[K,N]   with a fused epilogue.
//
// Roles (320 threads, one CTA per SM):
//   warps 0-7  epilogue: TMEM -> registers (tcgen05.ld), then store / reduce;
//              warp w reads TMEM lane quadrant w % 4, columns of half w / 4
//   warp 8     producer: TMA tile loads of A and B into a STAGES-deep ring
//   warp 9     MMA issuer: one elected lane issues tcgen05.mma, commits to mbarriers
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue
// of one output tile overlaps the main loop of the next.  Work units are
// (m tile, n tile, k slice) triples handed out round-robin; split-K slices
// reduce into fp32 with vector atomics.
//
// Operand layouts: A is K-major ([M][lda], K contiguous) or MN-major
// ([K][lda], M contiguous); B is K-major ([N][ldb]) or MN-major ([K][ldb]).
// All tiles use the 128-byte swizzle; K blocks are 64 elements wide.
#include <stdio.h>

#include "frnnt_common.cuh"
#include "frnnt_internal.h"
#include "sm100.cuh"

namespace frnnt {

using namespace sm100;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
// warps 0-7 epilogue (two per TMEM lane quadrant, each half of the tile's
// columns), warp 8 TMA producer, warp 9 MMA issuer
// Warp roles (EW = epilogue warps, 8 or 16): warps 0 .. EW-1 epilogue (EW/4
// per TMEM lane quadrant, each a 4/EW share of a tile's columns), warp EW the
// TMA producer, warp EW+1 the MMA issuer.  The d_hidden GEMM, whose epilogue
// (tanh' from F and G, segment sums) outweighs its MMAs, runs with 16
// epilogue warps so that each scheduler has four to hide the epilogue's load,
// MUFU and shuffle latencies (medium: 0.406 -> 0.390 ms); the other epilogues
// keep 8 (more registers per thread).
constexpr int threads_of(int EW) { return EW * 32 + 64; }

struct GemmParams {
  int M, N, K;
  int m_tiles, n_tiles, k_splits, kblocks;
  int epi;
  float* out_f32;
  __nv_bfloat16* out_bf16;
  long long ldo;
  int32_t* status;
  const int* dyn_count;
  int dyn_base, dyn_scale, dyn_dim;
  CellMap cells;
  int lose_first_load;   // test setting: no CTA loads (or announces) its first K block
};

// Effective problem after the optional device-side limit on M or K.
struct Eff {
  int M, m_tiles, kblocks, per;
};

__device__ __forceinline__ Eff eff_of(const GemmParams& p, bool early = false) {
  Eff e;
  e.M = p.M;
  e.kblocks = p.kblocks;
  if (p.dyn_count) {
    const int cnt = early ? tile_count_early(p.dyn_count) : __ldg(p.dyn_count);
    long long v = ((long long)cnt - p.dyn_base) * p.dyn_scale;
    if (v < 0) v = 0;
    if (p.dyn_dim == 1) e.M = (int)min((long long)p.M, v);
    else e.kblocks = (int)min((long long)p.kblocks, (v + 63) / 64);
  }
  e.m_tiles = (e.M + 127) / 128;
  e.per = (e.kblocks + p.k_splits - 1) / p.k_splits;
  return e;
}

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TILES_BYTES = STAGES * STAGE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int TOTAL = TILES_BYTES + BAR_BYTES + 1024;   // + alignment slack
};

// Unit -> (m tile origin, n tile index, k block range); false when the unit
// has no work under the effective limits (every role skips it alike).
__device__ __forceinline__ bool unit_coords(int unit, const GemmParams& p, const Eff& e, int& m0, int& nt, int& kb0,
                                           int& kb1) {
  // raster: the n tiles of one m tile run back to back when m tiles dominate, so
  // the A panel is fetched from DRAM once and re-read from L2 (k slices outermost)
  int mt;
  const int mn = unit % (p.m_tiles * p.n_tiles);
  const int ks = unit / (p.m_tiles * p.n_tiles);
  if (p.m_tiles >= p.n_tiles) {
    nt = mn % p.n_tiles;
    mt = mn / p.n_tiles;
  } else {
    mt = mn % p.m_tiles;
    nt = mn / p.m_tiles;
  }
  m0 = mt * BM;
  kb0 = ks * e.per;
  kb1 = min(e.kblocks, kb0 + e.per);
  return mt < e.m_tiles && kb0 < kb1;
}

__device__ __forceinline__ void epilogue_store(const GemmParams& p, int row, int col0, const uint32_t (&r)[32]) {
  if (p.epi == 0) {          // store fp32
    float4* dst = (float4*)(p.out_f32 + (size_t)row * p.ldo + col0);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                           __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
  } else if (p.epi == 1) {   // store bf16
    uint4* dst = (uint4*)(p.out_bf16 + (size_t)row * p.ldo + col0);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 v;
      v.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
      v.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
      v.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
      v.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
      dst[j] = v;
    }
  } else if (p.epi == 2) {   // fp32 reduce (split-K / accumulate)
    float* dst = p.out_f32 + (size_t)row * p.ldo + col0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      red_add_v4(dst + 4 * j, __uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
  }
}

// dtanh epilogue: out = acc * (1 - h^2), with h (bf16) read from out_bf16 into
// hv before the accumulator chunk is loaded from TMEM, and the result written
// back in place.
__device__ __forceinline__ void dtanh_load(const GemmParams& p, int row, int col0, uint4 (&hv)[4]) {
  const uint4* hp = (const uint4*)(p.out_bf16 + (size_t)row * p.ldo + col0);
#pragma unroll
  for (int j = 0; j < 4; ++j) hv[j] = hp[j];
}
__device__ __forceinline__ void dtanh_store(const GemmParams& p, int row, int col0, const uint32_t (&r)[32],
                                            const uint4 (&hv4)[4]) {
  uint4* hp = (uint4*)(p.out_bf16 + (size_t)row * p.ldo + col0);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 hv = hv4[j];
    const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&hw[q]);
      float2 hf = __bfloat1622float2(h2);
      float d0 = __uint_as_float(r[8 * j + 2 * q]) * (1.f - hf.x * hf.x);
      float d1 = __uint_as_float(r[8 * j + 2 * q + 1]) * (1.f - hf.y * hf.y);
      o[q] = pack_bf16x2(d0, d1);
    }
    hp[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Recompute-h dtanh epilogue: the F and G rows behind GEMM row `row` (null
// when the row is no lattice cell: its accumulator is zero, so is its result).
struct FgRows {
  const __nv_bfloat16* f;
  const __nv_bfloat16* g;
};
__device__ __forceinline__ FgRows fg_rows(const CellMap& m, int row) {
  const int4 td = m.tiles[m.tile0 + (row >> 7)];
  const int r = row & 127;
  const int b = td.x, t = td.y + r / m.UB;
  const int Tb = clampi(m.T_len[b], 1, m.T), Ub = clampi(m.U_len[b], 0, m.U);
  int u;
  bool valid;
  if (m.S) {
    const int j = r % m.UB;
    u = clampi(m.bounds[(size_t)b * m.T + min(t, Tb - 1)], 0, m.U) + j;
    valid = t < Tb && j < m.S && u <= Ub;
  } else {
    u = td.z + r % m.UB;
    valid = t < Tb && u <= Ub;
  }
  FgRows fr{nullptr, nullptr};
  if (valid) {
    fr.f = (const __nv_bfloat16*)m.F + ((size_t)b * m.T + t) * m.H;
    fr.g = (const __nv_bfloat16*)m.G + ((size_t)b * (m.U + 1) + u) * m.H;
  }
  return fr;
}
// Fused segment reduction (GEMM_EPI_DTANH_SEG).  The rows of a 128-row M tile
// are one cell tile: row r = frame t0 + r / UB and label (or band) position
// r % UB, so the UB consecutive lanes of a warp share a frame and, on the whole
// lattice, lanes UB apart share a label position.  A 32-column chunk of dpre is
// summed over a frame's lanes by recursive halving (each lane ends with 32/UB
// columns of the frame's sum) and over a label position's lanes likewise (UB
// columns each), then added to dF / dG with vector reductions.  On a pruned
// lattice the label positions differ per frame: every cell adds its own dG row.
struct SegRow {
  const __nv_bfloat16* f;   // F and G rows of the cell (null: no lattice cell, dpre = 0)
  const __nv_bfloat16* g;
  float* df;                // dF row of the lane's frame (null: the frame is outside the utterance)
  float* dg;                // dG row of the lane's label position (null: outside, or no cell when pruned)
};
__device__ __forceinline__ SegRow seg_row(const CellMap& m, int row, bool row_ok) {
  SegRow s{nullptr, nullptr, nullptr, nullptr};
  if (!row_ok) return s;
  const int4 td = m.tiles[m.tile0 + (row >> 7)];
  const int r = row & 127;
  const int b = td.x, t = td.y + r / m.UB;
  const int Tb = clampi(m.T_len[b], 1, m.T), Ub = clampi(m.U_len[b], 0, m.U);
  int u;
  bool uok;
  if (m.S) {
    const int j = r % m.UB;
    u = clampi(m.bounds[(size_t)b * m.T + min(t, Tb - 1)], 0, m.U) + j;
    uok = j < m.S && u <= Ub;
  } else {
    u = td.z + r % m.UB;
    uok = u <= Ub;
  }
  const bool tok = t < Tb;
  if (tok) s.df = m.dF + ((size_t)b * m.T + t) * m.H;
  if (uok && (m.S == 0 || tok)) s.dg = m.dG + ((size_t)b * (m.U + 1) + u) * m.H;
  if (tok && uok) {
    s.f = (const __nv_bfloat16*)m.F + ((size_t)b * m.T + t) * m.H;
    s.g = (const __nv_bfloat16*)m.G + ((size_t)b * (m.U + 1) + u) * m.H;
  }
  return s;
}

// One recursive-halving level over lanes s apart: of the first N values a
// lane keeps the upper half when (lane & s), the lower one otherwise, plus
// its partner's copy of that half.
template <int N, int A>
__device__ __forceinline__ void rs_level(float (&v)[A], int s, bool upper) {
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float give = upper ? v[i] : v[i + N / 2];
    const float keep = upper ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, give, s);
  }
}
// Sum over each group of G consecutive lanes (G <= N): v[0 .. N/G) becomes the
// sum of columns (N/G) (lane % G) + i.
template <int G, int N, int A>
__device__ __forceinline__ void rs_within(float (&v)[A], int lane) {
  if constexpr (G > 1) {
    rs_level<N>(v, G / 2, (lane & (G / 2)) != 0);
    rs_within<G / 2, N / 2>(v, lane);
  }
}
// Sum over the lanes congruent modulo G: v[0 .. N G/32) becomes the sum of
// columns (N G/32) (lane / G) + i.
template <int G, int N, int A, int S = 16>
__device__ __forceinline__ void rs_across(float (&v)[A], int lane) {
  if constexpr (S >= G) {
    rs_level<N>(v, S, (lane & S) != 0);
    rs_across<G, N / 2, A, S / 2>(v, lane);
  }
}
template <int NV, int A>
__device__ __forceinline__ void red_add_n(float* dst, const float (&v)[A]) {
  if constexpr (NV == 1) {
    red_add_f32(dst, v[0]);
  } else if constexpr (NV == 2) {
    red_add_v2(dst, v[0], v[1]);
  } else {
#pragma unroll
    for (int i = 0; i < NV; i += 4) red_add_v4(dst + i, v[i], v[i + 1], v[i + 2], v[i + 3]);
  }
}
// The sums of one chunk of N columns (N = 16 or 32) of dpre: into dF over the
// G lanes of a frame (G = the tile's label positions), into dG over the lanes
// of a label position (pruned lattice: each lane its own dG row).
template <int G, int N>
__device__ __forceinline__ void seg_chunk_g(const CellMap& m, const SegRow& sr, int col0, const float (&d)[N],
                                            int lane) {
  float v[N];
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = d[i];
  if constexpr (G <= N) {
    rs_within<G, N>(v, lane);
    if (sr.df) red_add_n<N / G>(sr.df + col0 + (N / G) * (lane & (G - 1)), v);
  } else {   // a 32-lane frame and 16 columns: sum each half-warp, then the halves
    rs_within<N, N>(v, lane);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 16);
    if (sr.df && lane < N) red_add_f32(sr.df + col0 + lane, v[0]);
  }
  if constexpr (G < 32) {
    if (m.S == 0) {
#pragma unroll
      for (int i = 0; i < N; ++i) v[i] = d[i];
      rs_across<G, N>(v, lane);
      if (sr.dg) red_add_n<N * G / 32>(sr.dg + col0 + (N * G / 32) * (lane / G), v);
      return;
    }
  }
  if (sr.dg) red_add_n<N>(sr.dg + col0, d);
}
// dpre = acc * tanh'(F + G) of the lane's row (0 when it is no cell), then the
// sums; sv4 holds the derivative (bf16, from dtanh_from_fg).  Every lane of the
// warp calls this for the same chunk (the shuffles need all).
template <int N>
__device__ __forceinline__ void seg_chunk(const CellMap& m, const SegRow& sr, int col0, const uint32_t (&r)[N],
                                          const uint4 (&sv4)[N / 8], int lane) {
  float d[N];
#pragma unroll
  for (int j = 0; j < N / 8; ++j) {
    const uint32_t sw[4] = {sv4[j].x, sv4[j].y, sv4[j].z, sv4[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 sf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sw[q]));
      d[8 * j + 2 * q] = sr.f ? __uint_as_float(r[8 * j + 2 * q]) * sf.x : 0.f;
      d[8 * j + 2 * q + 1] = sr.f ? __uint_as_float(r[8 * j + 2 * q + 1]) * sf.y : 0.f;
    }
  }
  switch (m.UB) {
    case 4: seg_chunk_g<4, N>(m, sr, col0, d, lane); break;
    case 8: seg_chunk_g<8, N>(m, sr, col0, d, lane); break;
    case 16: seg_chunk_g<16, N>(m, sr, col0, d, lane); break;
    default: seg_chunk_g<32, N>(m, sr, col0, d, lane); break;
  }
}

__device__ __forceinline__ uint32_t tanh_bf16x2_g(uint32_t x) {
  uint32_t y;
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// h (bf16, as the joint kernel and the h rows compute it) of 32 columns from
// col0, into hv (same layout as dtanh_load's: 4 x 8 bf16)
__device__ __forceinline__ void h_from_fg(const FgRows& fr, int col0, uint4 (&hv)[4]) {
  if (!fr.f) {
#pragma unroll
    for (int j = 0; j < 4; ++j) hv[j] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* fp = (const uint4*)(fr.f + col0);
  const uint4* gp = (const uint4*)(fr.g + col0);
  uint4 fv[4], gv[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    fv[j] = __ldg(fp + j);
    gv[j] = __ldg(gp + j);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __nv_bfloat162 a, c;
    uint32_t o[4];
    const uint32_t fw[4] = {fv[j].x, fv[j].y, fv[j].z, fv[j].w}, gw[4] = {gv[j].x, gv[j].y, gv[j].z, gv[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      a = *reinterpret_cast<const __nv_bfloat162*>(&fw[q]);
      c = *reinterpret_cast<const __nv_bfloat162*>(&gw[q]);
      __nv_bfloat162 sum = __hadd2(a, c);
      o[q] = tanh_bf16x2_g(*reinterpret_cast<uint32_t*>(&sum));
    }
    hv[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__device__ __forceinline__ float ex2_approx_g(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx_g(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// tanh'(x) = 1 - tanh(x)^2 = sech(x)^2 = 4e / (1 + e)^2 with e = exp(-2|x|) in
// (0, 1], in fp32 (two MUFU operations: exp2 and reciprocal, each within a few
// ulp).  Formed this way it keeps its relative accuracy where tanh saturates,
// which 1 - h^2 of a rounded h loses (h = 0.995 rounded to bf16 is off by up
// to 2^-9, the derivative there is 0.01).
__device__ __forceinline__ float sech2_f32(float x) {
  const float e = ex2_approx_g(-2.8853900817779268f * fabsf(x));   // 2 log2(e) |x|
  const float r2 = 2.f * rcp_approx_g(1.f + e);
  return e * r2 * r2;
}
// tanh'(F + G) of N columns (16 or 32) from col0 in bf16 pairs (F and G added
// in fp32), into sv (the layout of h_from_fg's output); zero when the row is no cell
template <int N>
__device__ __forceinline__ void dtanh_from_fg(const FgRows& fr, int col0, uint4 (&sv)[N / 8]) {
  if (!fr.f) {
#pragma unroll
    for (int j = 0; j < N / 8; ++j) sv[j] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* fp = (const uint4*)(fr.f + col0);
  const uint4* gp = (const uint4*)(fr.g + col0);
  uint4 fv[N / 8], gv[N / 8];
#pragma unroll
  for (int j = 0; j < N / 8; ++j) {
    fv[j] = __ldg(fp + j);
    gv[j] = __ldg(gp + j);
  }
#pragma unroll
  for (int j = 0; j < N / 8; ++j) {
    uint32_t o[4];
    const uint32_t fw[4] = {fv[j].x, fv[j].y, fv[j].z, fv[j].w}, gw[4] = {gv[j].x, gv[j].y, gv[j].z, gv[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&fw[q]));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[q]));
      o[q] = pack_bf16x2(sech2_f32(a.x + c.x), sech2_f32(a.y + c.y));
    }
    sv[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// dtanh epilogue: pull this thread's h row segment of a coming tile into L2
// while the tile's MMAs run, so the epilogue's reads do not wait on HBM.
__device__ __forceinline__ void dtanh_prefetch(const GemmParams& p, int row, int n0, int bn, int M) {
  if (row >= M) return;
  const __nv_bfloat16* base = (const __nv_bfloat16*)p.out_bf16 + (size_t)row * p.ldo;
  for (int c = n0; c < n0 + bn && c < p.N; c += 64) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + c));
}

template <int BN, int STAGES, bool A_MN, bool B_MN, int EW>
__global__ void __launch_bounds__(threads_of(EW), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  using S = GemmSmem<BN, STAGES>;
  constexpr int kEpiWarps = EW, kProdWarp = EW, kMmaWarp = EW + 1, kEpiParts = EW / 4;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + S::TILES_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_base_p = (uint32_t*)(tempty + 2);
  volatile int* abort_flag = (volatile int*)(tmem_base_p + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = p.m_tiles * p.n_tiles * p.k_splits;
  {
    // no work anywhere in the grid (a chunk past the device-built tile list):
    // every CTA sees the same limits and leaves before any set-up, after
    // waiting for the previous launch like every other launch of the call
    const Eff e0 = eff_of(p, true);
    if (e0.M <= 0 || e0.kblocks <= 0) {
      chain_wait();
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_base_p, 2 * BN);
    tmem_relinquish();
  }
  if (warp == kProdWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_p;
  // set-up done: from here on the previous launches' results are read
  chain_wait();
  const Eff eff = eff_of(p);

  if (warp == kProdWarp) {
    // ---------------------------------------------------------------- producer (warp polls, one lane issues)
    {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool lose = p.lose_first_load != 0;
      for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
        int m0, nt, kb0, kb1;
        if (!unit_coords(unit, p, eff, m0, nt, kb0, kb1)) continue;
        const int n0 = nt * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (lose) {
            lose = false;   // the stage's full barrier never completes: its consumer's wait runs out
          } else if (elect_one()) {
            uint8_t* sa = smem + s * S::STAGE_BYTES;
            uint8_t* sb = sa + S::A_BYTES;
            mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
            if (!A_MN) {
              tma_load_2d(sa, &tmA, &full[s], kb * BK, m0);
            } else {
              tma_load_2d(sa, &tmA, &full[s], m0, kb * BK);
              tma_load_2d(sa + 8192, &tmA, &full[s], m0 + 64, kb * BK);
            }
            if (!B_MN) {
              tma_load_2d(sb, &tmB, &full[s], kb * BK, n0);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 8192, &tmB, &full[s], n0 + 64 * j, kb * BK);
            }
          }
          __syncwarp();
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer (warp polls, one lane issues)
    {
      constexpr uint32_t idesc = idesc_bf16(BM, BN, A_MN, B_MN);
      int s = 0;
      uint32_t ph = 0;
      int acc_i = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
        int m0, nt, kb0, kb1;
        if (!unit_coords(unit, p, eff, m0, nt, kb0, kb1)) continue;
        const int a = acc_i & 1;
        const uint32_t aph = (acc_i >> 1) & 1;
        if (!warp_wait(&tempty[a], aph ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t dt = tbase + a * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          if (elect_one()) {
            const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
            const uint32_t sb = sa + S::A_BYTES;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint64_t ad = A_MN ? sdesc_sw128(sa + k * 2048, 8192, 1024) : sdesc_sw128(sa + k * 32, 16, 1024);
              const uint64_t bd = B_MN ? sdesc_sw128(sb + k * 2048, 8192, 1024) : sdesc_sw128(sb + k * 32, 16, 1024);
              mma_bf16_ss(dt, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
          }
          __syncwarp();
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok && elect_one()) mma_commit(&tfull[a]);
        __syncwarp();
        ++acc_i;
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (warps 0-7)
    int acc_i = 0;
    for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
      int m0, nt, kb0, kb1;
      if (!unit_coords(unit, p, eff, m0, nt, kb0, kb1)) continue;
      const int n0 = nt * BN;
      const int a = acc_i & 1;
      const uint32_t aph = (acc_i >> 1) & 1;
      const int q = warp & 3, half = warp >> 2;   // TMEM lane quadrant, column part
      const int row = m0 + q * 32 + lane;
      const bool row_ok = row < eff.M;
      if (p.epi == GEMM_EPI_DTANH && acc_i == 0)
        dtanh_prefetch(p, row, n0 + half * (BN / kEpiParts), BN / kEpiParts, eff.M);
      const FgRows fr = (p.epi == GEMM_EPI_DTANH_FG && row_ok) ? fg_rows(p.cells, row) : FgRows{nullptr, nullptr};
      const SegRow sr = p.epi == GEMM_EPI_DTANH_SEG ? seg_row(p.cells, row, row_ok) : SegRow{};
      if (!warp_wait(&tfull[a], aph, abort_flag)) break;   // warp-uniform: the epilogue uses warp-collective ops
      tc_fence_after();
      if constexpr (EW == 16) {
        // the d_hidden epilogue (the one launched with 16 epilogue warps) in
        // 16-column chunks: half the registers of 32-column ones, so the 96 a
        // thread gets at 576 threads hold it without spilling
#pragma unroll 1
        for (int c = half * (BN / (16 * kEpiParts)); c < (half + 1) * (BN / (16 * kEpiParts)); ++c) {
          const int col0 = n0 + c * 16;
          if (col0 >= p.N) break;   // the same for the whole warp; later chunks lie further right
          uint4 hv[2];
          dtanh_from_fg<16>(FgRows{sr.f, sr.g}, col0, hv);
          uint32_t r[16];
          tmem_ld16(tbase + ((uint32_t)(q * 32) << 16) + a * BN + c * 16, r);
          tmem_wait_ld();
          seg_chunk<16>(p.cells, sr, col0, r, hv, lane);   // whole warp, same chunk
        }
      } else {
#pragma unroll 1
        for (int c = half * (BN / (32 * kEpiParts)); c < (half + 1) * (BN / (32 * kEpiParts)); ++c) {
          uint32_t r[32];
          const int col0 = n0 + c * 32;
          const bool st = row_ok && col0 < p.N;
          uint4 hv[4];
          if (p.epi == GEMM_EPI_DTANH && st) dtanh_load(p, row, col0, hv);
          if (p.epi == GEMM_EPI_DTANH_FG && st) h_from_fg(fr, col0, hv);
          if (p.epi == GEMM_EPI_DTANH_SEG && col0 < p.N) dtanh_from_fg<32>(FgRows{sr.f, sr.g}, col0, hv);
          tmem_ld32(tbase + ((uint32_t)(q * 32) << 16) + a * BN + c * 32, r);
          tmem_wait_ld();
          if (p.epi == GEMM_EPI_DTANH_SEG) {
            if (col0 < p.N) seg_chunk<32>(p.cells, sr, col0, r, hv, lane);   // whole warp, same chunk
            continue;
          }
          if (!st) continue;
          if (p.epi == GEMM_EPI_DTANH || p.epi == GEMM_EPI_DTANH_FG) dtanh_store(p, row, col0, r, hv);
          else epilogue_store(p, row, col0, r);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
      ++acc_i;
      if (p.epi == GEMM_EPI_DTANH) {
        int nm0, nnt, nkb0, nkb1;
        if (unit + (int)gridDim.x < units && unit_coords(unit + gridDim.x, p, eff, nm0, nnt, nkb0, nkb1))
          dtanh_prefetch(p, nm0 + q * 32 + lane, nnt * BN + half * (BN / kEpiParts), BN / kEpiParts, eff.M);
      }
    }
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, 2 * BN);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, FRNNT_STATUS_TIMEOUT);
}


// ------------------------------------------------------------------ CTA-pair variant
// Two CTAs of a cluster share one M = 256 output tile: each stages its own 128
// rows of A and half of the B tile, the leader (rank 0) issues cta_group::2 MMAs
// that read both CTAs' shared memory, and each CTA's TMEM receives its 128 rows.
// Per CTA this halves the B-operand traffic of shared memory and of the L2.
template <int BN, int STAGES>
struct Gemm2Smem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = (BN / 2) * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TILES_BYTES = STAGES * STAGE_BYTES;
  static constexpr int TOTAL = TILES_BYTES + 256 + 1024;
};

__device__ __forceinline__ bool unit_coords2(int unit, const GemmParams& p, const Eff& e, int& m0, int& nt, int& kb0,
                                            int& kb1) {
  int mt;                                   // m tiles of 256 rows here
  const int mn = unit % (p.m_tiles * p.n_tiles);
  const int ks = unit / (p.m_tiles * p.n_tiles);
  if (p.m_tiles >= p.n_tiles) {
    nt = mn % p.n_tiles;
    mt = mn / p.n_tiles;
  } else {
    mt = mn % p.m_tiles;
    nt = mn / p.m_tiles;
  }
  m0 = mt * 256;
  kb0 = ks * e.per;
  kb1 = min(e.kblocks, kb0 + e.per);
  return m0 < e.M && kb0 < kb1;
}

template <int BN, int STAGES, bool A_MN, bool B_MN, int EW>
__global__ void __launch_bounds__(threads_of(EW), 1)
    gemm2_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  using S = Gemm2Smem<BN, STAGES>;
  constexpr int kEpiWarps = EW, kProdWarp = EW, kMmaWarp = EW + 1, kEpiParts = EW / 4;
  constexpr int HB = BN / 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + S::TILES_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_base_p = (uint32_t*)(tempty + 2);
  volatile int* abort_flag = (volatile int*)(tmem_base_p + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int units = p.m_tiles * p.n_tiles * p.k_splits;
  {
    // as in the one-CTA kernel: an empty launch leaves before any set-up or
    // cluster barrier (both CTAs of every pair alike)
    const Eff e0 = eff_of(p, true);
    if (e0.M <= 0 || e0.kblocks <= 0) {
      chain_wait();
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kEpiWarps);   // the epilogue warps of both CTAs of the pair
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_base_p, 2 * BN);
    tmem_relinquish_pair();
  }
  if (warp == kProdWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  cluster_sync();
  tc_fence_after();
  const uint32_t tbase = *tmem_base_p;
  // as in the one-CTA kernel: the previous launches' results are read from here on
  chain_wait();
  const Eff eff = eff_of(p);

  if (warp == kProdWarp) {
    // ---------------------------------------------------------------- producer (both CTAs; warp polls, one lane issues)
    {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      bool lose = p.lose_first_load != 0;
      for (int unit = pair; unit < units && ok; unit += npairs) {
        int m0, nt, kb0, kb1;
        if (!unit_coords2(unit, p, eff, m0, nt, kb0, kb1)) continue;
        const int ma = m0 + (int)rank * 128;
        const int nb = nt * BN + (int)rank * HB;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (lose) {
            lose = false;   // the leader's full barrier never completes: the MMA issuer's wait runs out
          } else if (elect_one()) {
            uint8_t* sa = smem + s * S::STAGE_BYTES;
            uint8_t* sb = sa + S::A_BYTES;
            const uint32_t fl = mapa_shared(smem_u32(&full[s]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * S::STAGE_BYTES);
            if (!A_MN) {
              tma_load_2d_pair(sa, &tmA, fl, kb * BK, ma);
            } else {
              tma_load_2d_pair(sa, &tmA, fl, ma, kb * BK);
              tma_load_2d_pair(sa + 8192, &tmA, fl, ma + 64, kb * BK);
            }
            if (!B_MN) {
              tma_load_2d_pair(sb, &tmB, fl, kb * BK, nb);
            } else {
#pragma unroll
              for (int j = 0; j < HB / 64; ++j) tma_load_2d_pair(sb + j * 8192, &tmB, fl, nb + 64 * j, kb * BK);
            }
          }
          __syncwarp();
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer (leader CTA only; warp polls, one lane issues)
    if (rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(256, BN, A_MN, B_MN);
      int s = 0;
      uint32_t ph = 0;
      int acc_i = 0;
      bool ok = true;
      for (int unit = pair; unit < units && ok; unit += npairs) {
        int m0, nt, kb0, kb1;
        if (!unit_coords2(unit, p, eff, m0, nt, kb0, kb1)) continue;
        const int a = acc_i & 1;
        const uint32_t aph = (acc_i >> 1) & 1;
        if (!warp_wait(&tempty[a], aph ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t dt = tbase + a * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          if (elect_one()) {
            const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
            const uint32_t sb = sa + S::A_BYTES;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint64_t ad = A_MN ? sdesc_sw128(sa + k * 2048, 8192, 1024) : sdesc_sw128(sa + k * 32, 16, 1024);
              const uint64_t bd = B_MN ? sdesc_sw128(sb + k * 2048, 8192, 1024) : sdesc_sw128(sb + k * 32, 16, 1024);
              mma_bf16_ss_pair(dt, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            }
            mma_commit_pair(&empty[s], 0x3);
          }
          __syncwarp();
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok && elect_one()) mma_commit_pair(&tfull[a], 0x3);
        __syncwarp();
        ++acc_i;
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (warps 0-7, both CTAs)
    int acc_i = 0;
    for (int unit = pair; unit < units; unit += npairs) {
      int m0, nt, kb0, kb1;
      if (!unit_coords2(unit, p, eff, m0, nt, kb0, kb1)) continue;
      const int n0 = nt * BN;
      const int a = acc_i & 1;
      const uint32_t aph = (acc_i >> 1) & 1;
      const int q = warp & 3, half = warp >> 2;   // TMEM lane quadrant, column part
      const int row = m0 + (int)rank * 128 + q * 32 + lane;
      const bool row_ok = row < eff.M;
      if (p.epi == GEMM_EPI_DTANH && acc_i == 0)
        dtanh_prefetch(p, row, n0 + half * (BN / kEpiParts), BN / kEpiParts, eff.M);
      const FgRows fr = (p.epi == GEMM_EPI_DTANH_FG && row_ok) ? fg_rows(p.cells, row) : FgRows{nullptr, nullptr};
      const SegRow sr = p.epi == GEMM_EPI_DTANH_SEG ? seg_row(p.cells, row, row_ok) : SegRow{};
      if (!warp_wait(&tfull[a], aph, abort_flag)) break;   // warp-uniform: the epilogue uses warp-collective ops
      tc_fence_after();
      if constexpr (EW == 16) {
        // the d_hidden epilogue (the one launched with 16 epilogue warps) in
        // 16-column chunks: half the registers of 32-column ones, so the 96 a
        // thread gets at 576 threads hold it without spilling
#pragma unroll 1
        for (int c = half * (BN / (16 * kEpiParts)); c < (half + 1) * (BN / (16 * kEpiParts)); ++c) {
          const int col0 = n0 + c * 16;
          if (col0 >= p.N) break;   // the same for the whole warp; later chunks lie further right
          uint4 hv[2];
          dtanh_from_fg<16>(FgRows{sr.f, sr.g}, col0, hv);
          uint32_t r[16];
          tmem_ld16(tbase + ((uint32_t)(q * 32) << 16) + a * BN + c * 16, r);
          tmem_wait_ld();
          seg_chunk<16>(p.cells, sr, col0, r, hv, lane);   // whole warp, same chunk
        }
      } else {
#pragma unroll 1
        for (int c = half * (BN / (32 * kEpiParts)); c < (half + 1) * (BN / (32 * kEpiParts)); ++c) {
          uint32_t r[32];
          const int col0 = n0 + c * 32;
          const bool st = row_ok && col0 < p.N;
          uint4 hv[4];
          if (p.epi == GEMM_EPI_DTANH && st) dtanh_load(p, row, col0, hv);
          if (p.epi == GEMM_EPI_DTANH_FG && st) h_from_fg(fr, col0, hv);
          if (p.epi == GEMM_EPI_DTANH_SEG && col0 < p.N) dtanh_from_fg<32>(FgRows{sr.f, sr.g}, col0, hv);
          tmem_ld32(tbase + ((uint32_t)(q * 32) << 16) + a * BN + c * 32, r);
          tmem_wait_ld();
          if (p.epi == GEMM_EPI_DTANH_SEG) {
            if (col0 < p.N) seg_chunk<32>(p.cells, sr, col0, r, hv, lane);   // whole warp, same chunk
            continue;
          }
          if (!st) continue;
          if (p.epi == GEMM_EPI_DTANH || p.epi == GEMM_EPI_DTANH_FG) dtanh_store(p, row, col0, r, hv);
          else epilogue_store(p, row, col0, r);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&tempty[a]), 0));   // only TMEM was read
      ++acc_i;
      if (p.epi == GEMM_EPI_DTANH) {
        int nm0, nnt, nkb0, nkb1;
        if (unit + npairs < units && unit_coords2(unit + npairs, p, eff, nm0, nnt, nkb0, nkb1))
          dtanh_prefetch(p, nm0 + (int)rank * 128 + q * 32 + lane, nnt * BN + half * (BN / kEpiParts),
                         BN / kEpiParts, eff.M);
      }
    }
  }

  __syncthreads();
  cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 2 * BN);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, FRNNT_STATUS_TIMEOUT);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

int g_lose_loads = 0;   // GEMM launches left whose first K block load is dropped (test setting)

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int BN, int STAGES, bool A_MN, bool B_MN, int EW = 8>
bool launch_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, int grid, cudaStream_t st) {
  using S = GemmSmem<BN, STAGES>;
  auto kern = gemm_tc_kernel<BN, STAGES, A_MN, B_MN, EW>;
  static bool attr[kDeviceSlots] = {};
  const int dev = current_device();
  if (!attr[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL) != cudaSuccess)
      return false;
    attr[dev] = true;
  }
  launch_k(kern, dim3(grid), dim3(threads_of(EW)), S::TOTAL, st, 1, ta, tb, p);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess;
}

template <int BN, int STAGES, bool A_MN, bool B_MN, int EW = 8>
bool launch2_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, int grid, cudaStream_t st) {
  using S = Gemm2Smem<BN, STAGES>;
  auto kern = gemm2_tc_kernel<BN, STAGES, A_MN, B_MN, EW>;
  static bool attr[kDeviceSlots] = {};
  const int dev = current_device();
  if (!attr[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL) != cudaSuccess)
      return false;
    attr[dev] = true;
  }
  const bool ok = launch_k(kern, dim3(grid), dim3(threads_of(EW)), S::TOTAL, st, 2, ta, tb, p) == cudaSuccess;
  note_launch();
  return ok && cudaPeekAtLastError() == cudaSuccess;
}

}  // namespace

// K slices of a split-K GEMM with mn output tiles on `workers` persistent CTAs
// (or CTA pairs), each taking units workers apart.  The launch lasts about
// rounds x (k blocks per unit + a unit's fixed cost: pipeline fill and the
// atomic epilogue), so the slice count minimising that is taken, the fewest on
// a tie.  A round that only a few workers reach costs as much as a full one:
// 12 tiles x 13 slices = 156 units on 74 pairs keep 8 pairs busy for a third
// round, where 6 slices fit one.  The fixed cost is taken as 64 k blocks, which
// favours fewer slices (fewer atomic epilogues) where the fill is about equal:
// on 40000 k blocks, 6 slices (one round) and 37 (six) measured the same.
int auto_splits(int mn, int workers, int kblocks) {
  if (mn <= 0 || workers <= 0 || kblocks <= 1) return 1;
  constexpr long long kUnitCost = 64;
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= kblocks; ++s) {
    const int per = (kblocks + s - 1) / s;
    const int real = (kblocks + per - 1) / per;   // slices after rounding each to whole k blocks
    if (real != s) continue;
    const long long units = (long long)mn * real;
    const long long rounds = (units + workers - 1) / workers;
    const long long cost = rounds * (per + kUnitCost);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = real;
    }
    if (rounds > 16) break;   // more slices only add rounds
  }
  return best;
}

bool make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_elems,
                       uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int gemm_tc(const GemmTcArgs& g, cudaStream_t st) {
  // shape rules of the tensor-core GEMM: 16-byte aligned rows and N a multiple of 32
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return FRNNT_OK;
  if ((g.lda % 8) || (g.ldb % 8) || (g.N % 32)) return FRNNT_ERR_DIMS;
  if ((g.epi == GEMM_EPI_STORE_F32 || g.epi == GEMM_EPI_RED_F32) && (g.ldo % 4 || !g.out_f32)) return FRNNT_ERR_DIMS;
  if ((g.epi == GEMM_EPI_STORE_BF16 || g.epi == GEMM_EPI_DTANH || g.epi == GEMM_EPI_DTANH_FG) &&
      (g.ldo % 8 || !g.out_bf16))
    return FRNNT_ERR_DIMS;
  if (g.epi == GEMM_EPI_DTANH_SEG && (!g.cells.tiles || !g.cells.F || !g.cells.G || !g.cells.dF || !g.cells.dG))
    return FRNNT_ERR_DIMS;
  if (((uintptr_t)g.A | (uintptr_t)g.B | (uintptr_t)g.out_f32 | (uintptr_t)g.out_bf16) & 15u) return FRNNT_ERR_ALIGN;
  // variants 2 / 3: 256-wide N tiles even when N is not a multiple of 256 (the
  // last tile's missing B rows are zero-filled by TMA; its extra columns are
  // computed and not stored), one CTA / CTA pairs
  // (automatic: also for tall GEMMs with N > 512 and N % 256 >= 128, e.g. the
  // d_hidden GEMM at H = 640, where the wider tiles' halved L2 traffic outweighs
  // the last tile's extra columns; short ones such as the projections keep 128)
  const bool wide = (g.N % 256 == 0 && g.N >= 256) || (g.M >= 65536 && g.N > 512 && g.N % 256 >= 128);
  const int BN = (wide || g.variant >= 2) ? 256 : 128;
  // CTA pairs (M = 256 per MMA) for 256-wide N tiles on problems with enough rows
  const bool pair = g.variant == 1 || g.variant == 3 || (g.variant < 0 && g.M >= 512 && BN == 256);
  CUtensorMap ta, tb;
  bool ok;
  if (!g.a_mn) ok = make_tmap_bf16_2d(&ta, g.A, g.K, g.M, (uint64_t)g.lda, 64, 128);
  else ok = make_tmap_bf16_2d(&ta, g.A, g.M, g.K, (uint64_t)g.lda, 64, 64);
  if (!ok) return FRNNT_ERR_CUDA;
  const int b_rows = pair ? BN / 2 : BN;
  if (!g.b_mn) ok = make_tmap_bf16_2d(&tb, g.B, g.K, g.N, (uint64_t)g.ldb, 64, b_rows);
  else ok = make_tmap_bf16_2d(&tb, g.B, g.b_inner > 0 && g.b_inner < g.N ? g.b_inner : g.N, g.K, (uint64_t)g.ldb,
                              64, 64);
  if (!ok) return FRNNT_ERR_CUDA;
  GemmParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.m_tiles = (g.M + (pair ? 255 : 127)) / (pair ? 256 : 128);
  p.n_tiles = (g.N + BN - 1) / BN;
  p.kblocks = (g.K + BK - 1) / BK;
  int splits = g.k_splits;
  if (splits == 0 && g.epi == GEMM_EPI_RED_F32)
    splits = auto_splits(p.m_tiles * p.n_tiles, pair ? sm_count() / 2 : sm_count(), p.kblocks);
  if (splits < 1) splits = 1;
  if (splits > p.kblocks) splits = p.kblocks;
  if (splits > 1 && g.epi != GEMM_EPI_RED_F32) return FRNNT_ERR_UNSUPPORTED;
  // every split must own at least one k block
  const int per = (p.kblocks + splits - 1) / splits;
  splits = (p.kblocks + per - 1) / per;
  p.k_splits = splits;
  p.epi = g.epi;
  p.out_f32 = g.out_f32;
  p.out_bf16 = (__nv_bfloat16*)g.out_bf16;
  p.ldo = g.ldo;
  p.status = g.status;
  p.dyn_count = g.dyn_count;
  p.dyn_base = g.dyn_base;
  p.dyn_scale = g.dyn_scale;
  p.dyn_dim = g.dyn_dim;
  p.cells = g.cells;
  p.lose_first_load = 0;
  if (g_lose_loads > 0) {
    --g_lose_loads;
    p.lose_first_load = 1;
  }
  const int units = p.m_tiles * p.n_tiles * p.k_splits;
  const bool seg = g.epi == GEMM_EPI_DTANH_SEG;   // 16 epilogue warps
  bool launched;
  if (pair) {
    const int npairs = units < sm_count() / 2 ? units : sm_count() / 2;
    const int grid = 2 * npairs;
    if (BN == 256) {
      if (!g.a_mn && !g.b_mn) launched = launch2_t<256, 6, false, false>(ta, tb, p, grid, st);
      else if (!g.a_mn && g.b_mn)
        // the d_hidden GEMM with a 4-stage ring: measured faster than 5 or 6
        // (medium 0.381 -> 0.367 ms, long 3.26 -> 3.11 ms; 3 stages: 0.391),
        // the shared memory left over going to L1, which holds the epilogue's
        // F and G rows
        launched = seg ? launch2_t<256, 4, false, true, 16>(ta, tb, p, grid, st)
                       : launch2_t<256, 6, false, true>(ta, tb, p, grid, st);
      else if (g.a_mn && !g.b_mn) launched = launch2_t<256, 6, true, false>(ta, tb, p, grid, st);
      else launched = launch2_t<256, 6, true, true>(ta, tb, p, grid, st);
    } else {
      if (!g.a_mn && !g.b_mn) launched = launch2_t<128, 8, false, false>(ta, tb, p, grid, st);
      else if (!g.a_mn && g.b_mn)
        launched = seg ? launch2_t<128, 8, false, true, 16>(ta, tb, p, grid, st)
                       : launch2_t<128, 8, false, true>(ta, tb, p, grid, st);
      else if (g.a_mn && !g.b_mn) launched = launch2_t<128, 8, true, false>(ta, tb, p, grid, st);
      else launched = launch2_t<128, 8, true, true>(ta, tb, p, grid, st);
    }
    return launched ? FRNNT_OK : FRNNT_ERR_CUDA;
  }
  const int grid = units < sm_count() ? units : sm_count();
  if (BN == 256) {
    if (!g.a_mn && !g.b_mn) launched = launch_t<256, 4, false, false>(ta, tb, p, grid, st);
    else if (!g.a_mn && g.b_mn)
      launched = seg ? launch_t<256, 4, false, true, 16>(ta, tb, p, grid, st)
                     : launch_t<256, 4, false, true>(ta, tb, p, grid, st);
    else if (g.a_mn && !g.b_mn) launched = launch_t<256, 4, true, false>(ta, tb, p, grid, st);
    else launched = launch_t<256, 4, true, true>(ta, tb, p, grid, st);
  } else {
    if (!g.a_mn && !g.b_mn) launched = launch_t<128, 6, false, false>(ta, tb, p, grid, st);
    else if (!g.a_mn && g.b_mn)
      launched = seg ? launch_t<128, 6, false, true, 16>(ta, tb, p, grid, st)
                     : launch_t<128, 6, false, true>(ta, tb, p, grid, st);
    else if (g.a_mn && !g.b_mn) launched = launch_t<128, 6, true, false>(ta, tb, p, grid, st);
    else launched = launch_t<128, 6, true, true>(ta, tb, p, grid, st);
  }
  return launched ? FRNNT_OK : FRNNT_ERR_CUDA;
}

int lose_gemm_loads(int n) {
  const int prev = g_lose_loads;
  g_lose_loads = n < 0 ? 0 : n;
  return prev;
}

}  // namespace frnnt
