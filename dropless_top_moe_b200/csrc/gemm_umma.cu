// Persistent tcgen05 / TMEM grouped GEMM for bf16 expert FFNs (sm_100a).
//
// The expert FFN of the dropless layer is a set of per-expert GEMMs over
// variable-size row groups ("MegaBlocks - architecture", sec. 2.1, grouped
// path gmm -> act -> gmm; sec. 4: backward through the same grouping).  Every
// expert's rows are padded to multiples of 128, so each 128-row M tile lies in
// one expert; the tile -> expert map is a search in the device-side
// padded_bins, so the schedule never needs the counts on the host (the
// MegaBlocks grouped path copies them to the host; MoonEP sec. 02 argues for
// static shapes without host sync).
//
// One CTA (or one CTA pair, cta_group::2) per SM, 10 warps (18 in the
// single-CTA 256-row plain-store GEMMs, whose epilogue has 16 warps):
//   warp 0      producer: A and B tiles by TMA into a STAGES-deep smem ring,
//               one 64-deep k block per stage (two for a CTA pair, whose
//               MN-major operands come in 128-deep boxes)
//               (optionally A rows gathered from x with tile::gather4)
//   warp 1      TMEM allocator and MMA issuer (one thread): tcgen05.mma per
//               16-deep k step, fp32 accumulators in TMEM, double-buffered
//               where two accumulator sets fit so the epilogue of tile i
//               overlaps the main loop of tile i+1
//   warps 2..   epilogue, two (four) warps per TMEM lane quarter: tcgen05.ld rows ->
//               registers -> fused math -> global, 32 x 32 chunks through
//               a per-warp shared-memory scratch (TMA stores, or coalesced
//               64-byte row segments for the weight gradients)
// Tile shapes: BN output columns; MT 128-row tiles per CTA; CG = 2 pairs two
// CTAs on one M = 256 MMA (each CTA holds its 128 rows and half of B's
// columns); an expert's odd last tile runs as an M = 128 pair MMA, except
// that experts of a single tile can be left to a second, single-CTA launch
// (Params::single_mode) where many of them would each cost a pair unit.
// Schedules
//   ROWS   C[rows of group e, :] = A[rows, :] * B_e   (forward, dgrad)
//   WGRAD  C_e = A[group e rows, :]^T * B[group e rows, :]   (weight grads;
//          K = the group's padded rows, zero rows contribute nothing)
//   DENSE  C = A * B over plain row tiles x column tiles (the dense router
//          backward's D * W_r^T)
// Every accumulation runs in a fixed order (k-steps in sequence, no split-K
// across CTAs), so results are bitwise reproducible.  Every wait is bounded
// (status bit MOE_DEVERR_TIMEOUT); no TMA load uses multicast.
#include <cuda.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"
#include "umma.cuh"

namespace moe {
namespace umma {

constexpr int BM = 128;
constexpr int BK = 64;              // one 128-byte swizzle row of bf16
// Epilogue warps per CTA: 8 (two per TMEM lane quarter, splitting the
// columns), or 16 for the single-CTA 256-row plain-store GEMMs, whose one
// accumulator set keeps the epilogue off the main loop's critical path only
// if it drains fast (four warps per lane quarter, one scratch buffer each)
constexpr int kEpiWarps = 8;
constexpr uint64_t kTimeoutNs = 4000000000ull;
// Most M units per raster group (groups never span two experts, see
// get_tile): 8 units of up to 256 rows, so an expert of up to 2048 rows streams
// each weight column panel once
constexpr int kGroupM = 8;

enum Sched { SCHED_ROWS = 0, SCHED_WGRAD = 1, SCHED_DENSE = 2 };
enum Epi { EPI_SWIGLU = 0, EPI_STORE = 1, EPI_SWIGLU_BWD = 2, EPI_WGRAD = 3, EPI_WGRAD_PAIR = 4,
           EPI_ROUTER_DX = 6 };
enum Split { SPLIT_NONE = 0, SPLIT_K = 1, SPLIT_N = 2 };

struct Params {
  CUtensorMap ta0, ta1, tb0, tb1;
  CUtensorMap to0, to1, to2;   // outputs of the TMA-store epilogues (32 x 32 boxes)
  const int32_t* padded_bins;
  int E;
  int64_t P;          // rows of row-indexed buffers (ROWS/WGRAD) or tokens (DENSE)
  int kdim;           // ROWS/DENSE: K extent (both halves for SPLIT_K)
  int ksplit;         // SPLIT_K: first k of the second operand pair
  int n_mma;          // MMA N (== BN except DENSE, where it is E)
  int n_tiles;        // tiles along N
  int m_tiles_w;      // WGRAD: tiles along M
  int group_m;        // ROWS: M units per raster group
  // ROWS: which experts the launch covers: 0 all, 1 those of two or more
  // 128-row tiles, 2 those of exactly one (each then one unit; UNIT = 1)
  int single_mode;
  // Gathered A (GA kernels): ta0 maps the token matrix [g_N, kdim or M] with
  // one-row boxes; padded row r of expert e holds token
  // g_indices[g_bins[e-1] + r - padded_bins[e-1]] / g_K, pad rows read zeros
  const int32_t* g_indices;
  const int32_t* g_bins;
  int g_K;
  int g_N;
  __nv_bfloat16* out0;
  __nv_bfloat16* out1;
  __nv_bfloat16* out2;
  const __nv_bfloat16* aux0;
  const __nv_bfloat16* aux1;
  int64_t ldo;        // row stride (elements) of out* / aux*
  int64_t out_estride;// WGRAD: elements between consecutive experts' outputs
  int* status;
};

struct Tile {
  int e;
  int64_t row0;    // ROWS/DENSE: first A row; WGRAD: first contraction row
  int m0;          // WGRAD: first output row (of the weight gradient)
  int n0;          // first output column (per output matrix)
  int nkb;         // k-blocks of BK
  int halves;      // 128-row halves of the M tile in use (1 or 2)
};

// Compile-time shape of one kernel instance.  MT = 128-row M halves per tile:
// with MT = 2 two M=128 MMAs share every B tile, so a 256 x BN tile moves
// (2*128 + BN) rows of operands per k-step instead of (128 + BN) per half.
template <int BN, int MT, int CG = 1>
struct Shape {
  static constexpr int A_BYTES = MT * BM * BK * 2;
  static constexpr int B_BYTES = (CG == 2 ? BN / 2 : BN) * BK * 2;   // a pair splits B's columns
  static constexpr int SUB_BYTES = A_BYTES + B_BYTES;                 // one BK-deep k block
  // k blocks per pipeline stage: a pair's four M = 256 MMAs per k block take
  // less time than the issuing thread's per-stage work (barrier wait, commit,
  // four issues), so a pair stage holds two k blocks
  static constexpr int KSUB = CG == 2 ? 2 : 1;
  static constexpr int STAGE_BYTES = KSUB * SUB_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
  static constexpr int ACC_COLS = MT * BN;                       // one accumulator set
  static constexpr int ACC_BUFS = 2 * ACC_COLS <= 512 ? 2 : 1;   // double-buffer when it fits
  static constexpr int USED_COLS = ACC_BUFS * ACC_COLS;
  static constexpr uint32_t TMEM_COLS =
      USED_COLS <= 32 ? 32 : (USED_COLS <= 64 ? 64 : (USED_COLS <= 128 ? 128 : (USED_COLS <= 256 ? 256 : 512)));
  static constexpr int N_BARS = 2 * STAGES + 2 * ACC_BUFS + 1;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + 1024 + 8 * N_BARS + 16 + 4 * 260;
  // 128-row tiles per scheduling unit: MT per CTA, times 2 for a pair
  static constexpr int UNIT = MT * CG;
};


// Number of M units for the ROWS schedule: groups of UNIT consecutive 128-row
// tiles of the same expert (the last unit of an expert may hold fewer).
// s_unit_start[e] = first unit of expert e; s_unit_start[E] = all units.
__device__ __forceinline__ int64_t rows_units(const int32_t* s_unit_start, int E) { return s_unit_start[E]; }

template <int SCHED, int BN, int UNIT, int EPI>
__device__ __forceinline__ int64_t total_tiles(const Params& p, const int32_t* s_unit_start) {
  if constexpr (SCHED == SCHED_ROWS) {
    return rows_units(s_unit_start, p.E) * p.n_tiles;
  } else if constexpr (SCHED == SCHED_WGRAD) {
    return (int64_t)p.E * p.m_tiles_w * p.n_tiles;
  } else {
    return cdiv(p.P, BM) * (p.n_tiles > 1 ? p.n_tiles : 1);
  }
}

template <int SCHED, int BN, int UNIT, int EPI>
__device__ __forceinline__ Tile get_tile(const Params& p, int64_t t, const int32_t* s_unit_start) {
  constexpr int NOUT = (EPI == EPI_SWIGLU || EPI == EPI_WGRAD_PAIR) ? BN / 2 : BN;
  Tile tl;
  if constexpr (SCHED == SCHED_ROWS) {
    // Raster aligned to experts: expert e owns tiles [s_unit_start[e] * n,
    // s_unit_start[e + 1] * n) of the n column tiles; its units are cut into
    // nearly equal groups of at most group_m, and a group's tiles run
    // unit-fastest, so each weight column panel serves all the group's units
    // back to back and no group mixes two experts' weights (on B200 this
    // takes GEMM1's DRAM traffic from 1.52x to 1.06x its algorithmic bytes).
    const int64_t n = p.n_tiles;
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {                                  // last e owning tiles <= t
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)s_unit_start[mid] * n <= t) lo = mid; else hi = mid - 1;
    }
    tl.e = lo;
    const int64_t units_e = s_unit_start[lo + 1] - s_unit_start[lo];
    const int64_t local = t - (int64_t)s_unit_start[lo] * n;
    const int64_t nch = (units_e + p.group_m - 1) / p.group_m;   // groups of the expert
    const int64_t cs = (units_e + nch - 1) / nch;                // units per group (last: fewer)
    const int64_t c = local / (cs * n);
    const int64_t gm = (c == nch - 1) ? units_e - cs * (nch - 1) : cs;
    const int64_t lg = local - c * cs * n;
    const int64_t k = c * cs + lg % gm;                          // unit within the expert
    const int64_t nt = lg / gm;
    const int64_t pstart = tl.e ? p.padded_bins[tl.e - 1] : 0;
    int64_t pend = p.padded_bins[tl.e];
    if (pend > p.P) pend = p.P;
    const int64_t ntile_e = pend > pstart ? (pend - pstart) / BM : 0;
    tl.row0 = pstart + k * UNIT * BM;
    tl.halves = (int)((ntile_e - UNIT * k) >= UNIT ? UNIT : (ntile_e - UNIT * k));
    tl.m0 = 0;
    tl.n0 = (int)(nt * NOUT);
    tl.nkb = p.kdim / BK;
  } else if constexpr (SCHED == SCHED_WGRAD) {
    const int64_t per_e = (int64_t)p.m_tiles_w * p.n_tiles;
    tl.e = (int)(t / per_e);
    const int64_t r = t - (int64_t)tl.e * per_e;
    tl.m0 = (int)((r / p.n_tiles) * BM * UNIT);
    tl.n0 = (int)((r % p.n_tiles) * NOUT);
    const int64_t lo = tl.e ? p.padded_bins[tl.e - 1] : 0;
    int64_t hi = p.padded_bins[tl.e];
    if (hi > p.P) hi = p.P;
    tl.row0 = lo;
    tl.nkb = hi > lo ? (int)((hi - lo) / BK) : 0;
    tl.halves = UNIT;
  } else {
    // plain row tiles x n_tiles column tiles (the router: one column tile)
    const int64_t nt = p.n_tiles > 1 ? p.n_tiles : 1;
    tl.e = 0;
    tl.row0 = (t / nt) * BM;
    tl.m0 = 0;
    tl.n0 = (int)((t % nt) * BN);
    tl.nkb = p.kdim / BK;
    tl.halves = 1;
  }
  return tl;
}

__device__ __forceinline__ void store_row_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                      pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void load_row_bf16x32(const __nv_bfloat16* src, float* v) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = s[q];
    v[8 * q + 0] = bf16_lo(w.x); v[8 * q + 1] = bf16_hi(w.x);
    v[8 * q + 2] = bf16_lo(w.y); v[8 * q + 3] = bf16_hi(w.y);
    v[8 * q + 4] = bf16_lo(w.z); v[8 * q + 5] = bf16_hi(w.z);
    v[8 * q + 6] = bf16_lo(w.w); v[8 * q + 7] = bf16_hi(w.w);
  }
}

// Shared-memory scratch per epilogue warp: 32 rows x 64 bytes (one 32-column
// chunk of bf16) per buffer.
constexpr int kStoreBuf = 32 * 64;

// How an epilogue writes its rows.  A TMEM load gives each lane one row, so a
// store straight from registers sends 32 rows per warp instruction.
//   STORE_TMA        the chunk goes through one of two scratch buffers to a
//                    TMA store (SwiGLU, SwiGLU backward, plain stores:
//                    measured 4-9 % faster per GEMM on B200 than storing
//                    from registers or through the warp)
//   STORE_COALESCED  through one scratch buffer to 64-byte row segments by
//                    the warp (the weight gradients: TMA stores measured 5 %
//                    slower there)
//   STORE_DIRECT     straight from registers (the dense router dx)
enum StoreMode { STORE_DIRECT = 0, STORE_COALESCED = 1, STORE_TMA = 2 };
template <int EPI>
__host__ __device__ constexpr int store_mode() {
  return (EPI == EPI_STORE || EPI == EPI_SWIGLU_BWD || EPI == EPI_SWIGLU) ? STORE_TMA
         : (EPI == EPI_WGRAD || EPI == EPI_WGRAD_PAIR) ? STORE_COALESCED
                                                       : STORE_DIRECT;
}
template <int EPI>
__host__ __device__ constexpr int scratch_bytes() {
  return store_mode<EPI>() == STORE_TMA ? 2 * kStoreBuf
         : store_mode<EPI>() == STORE_COALESCED || EPI == EPI_SWIGLU_BWD ? kStoreBuf : 0;
}

// TMA store of a warp's 32 x 32 bf16 chunk: lane i holds row i's 32 values v;
// (x, y) = (first column, first row) of the chunk in map m.  The chunk is
// written to one of the warp's two scratch buffers (nb alternates) in the
// 64-byte swizzle layout the map expects -- 16-byte piece q of row r at
// position q ^ ((r >> 1) & 3), which also keeps the writes free of bank
// conflicts -- and one lane hands it to the TMA unit.  Before a buffer is
// rewritten, the store that used it two chunks earlier must have read it.
// Lane i's row i of a 32 x 32 bf16 chunk into scratch buffer buf, in the
// 64-byte swizzle layout of the output maps.
__device__ __forceinline__ void stage_chunk(uint32_t buf, int lane, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t a = buf + (uint32_t)(lane * 64) + ((uint32_t)(q ^ ((lane >> 1) & 3)) << 4);
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(pack_bf16x2(v[8 * q + 0], v[8 * q + 1])),
                 "r"(pack_bf16x2(v[8 * q + 2], v[8 * q + 3])), "r"(pack_bf16x2(v[8 * q + 4], v[8 * q + 5])),
                 "r"(pack_bf16x2(v[8 * q + 6], v[8 * q + 7]))
                 : "memory");
  }
}

__device__ __forceinline__ void store_chunk_tma(uint32_t scratch, int& nb, int lane, const CUtensorMap* m,
                                                int x, int y, const float* v) {
  const uint32_t buf = scratch + (uint32_t)(nb * kStoreBuf);
  nb ^= 1;
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t a = buf + (uint32_t)(lane * 64) + ((uint32_t)(q ^ ((lane >> 1) & 3)) << 4);
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(pack_bf16x2(v[8 * q + 0], v[8 * q + 1])),
                 "r"(pack_bf16x2(v[8 * q + 2], v[8 * q + 3])), "r"(pack_bf16x2(v[8 * q + 4], v[8 * q + 5])),
                 "r"(pack_bf16x2(v[8 * q + 6], v[8 * q + 7]))
                 : "memory");
  }
  fence_proxy_async();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(m, buf, x, y);
    bulk_commit();
  }
}

// Store a warp's 32 x 32 bf16 chunk: lane i holds row i's 32 values v; base
// points at the chunk's first element (row 0), ld is the row stride.  Storing
// straight from registers would send 32 rows (32 write requests) per warp
// store; instead the chunk goes through the warp's scratch and leaves as
// 64-byte row segments, 4 lanes per row and 8 rows per store.  A row's four
// 16-byte pieces sit at positions q ^ ((row >> 1) & 3), which keeps both the
// writes (a row per lane) and the reads (4 lanes per row) free of bank
// conflicts.
__device__ __forceinline__ void store_chunk_coalesced(uint32_t scratch, int lane, __nv_bfloat16* base,
                                                      int64_t ld, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t a = scratch + (uint32_t)(lane * 64) + ((uint32_t)(q ^ ((lane >> 1) & 3)) << 4);
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(pack_bf16x2(v[8 * q + 0], v[8 * q + 1])),
                 "r"(pack_bf16x2(v[8 * q + 2], v[8 * q + 3])), "r"(pack_bf16x2(v[8 * q + 4], v[8 * q + 5])),
                 "r"(pack_bf16x2(v[8 * q + 6], v[8 * q + 7]))
                 : "memory");
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = 8 * i + (lane >> 2), q = lane & 3;
    const uint32_t a = scratch + (uint32_t)(rr * 64) + ((uint32_t)(q ^ ((rr >> 1) & 3)) << 4);
    uint4 w;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w) : "r"(a) : "memory");
    st_v4(base + rr * ld + 8 * q, w);
  }
  __syncwarp();
}

// The reverse for loads: w[i] holds the 16-byte piece (lane & 3) of row
// 8i + lane / 4 of a 32 x 32 bf16 chunk, read as 64-byte row segments; after
// the exchange through the warp's scratch, lane i holds row i's 32 values.
__device__ __forceinline__ void rows_from_coalesced(uint32_t scratch, int lane, const uint4 (&w)[4], float* v) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = 8 * i + (lane >> 2), q = lane & 3;
    const uint32_t a = scratch + (uint32_t)(rr * 64) + ((uint32_t)(q ^ ((rr >> 1) & 3)) << 4);
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(w[i].x), "r"(w[i].y), "r"(w[i].z),
                 "r"(w[i].w)
                 : "memory");
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t a = scratch + (uint32_t)(lane * 64) + ((uint32_t)(q ^ ((lane >> 1) & 3)) << 4);
    uint4 u;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(a) : "memory");
    Vec<__nv_bfloat16>::to_float(u, v + 8 * q);
  }
  __syncwarp();
}

// Epilogue of one 128-row half: TMEM columns [tacc, tacc + BN) of this
// thread's row -> fused math -> global memory (store_mode<EPI>).  scratch:
// this warp's shared memory (scratch_bytes<EPI>(), or one buffer when NPART
// is 4); nb: the warp's next TMA-store buffer, carried across calls.
template <int BN, int SCHED, int EPI, int NPART = 2>
__device__ __forceinline__ void epilogue_half(const Params& p, const Tile& tl, uint32_t tacc, int row,
                                              int part, uint32_t scratch, int& nb) {
  const int64_t grow = tl.row0 + row;                 // ROWS/DENSE global row
  const int lane = row & 31;
  const int64_t row_base = grow - lane;               // the warp's first row (ROWS/DENSE)
  const int yb = (int)row_base;
  // the NPART warps of a lane quarter split the columns
  constexpr int NC = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
  static_assert((NC / NPART) % 32 == 0, "whole 32-column chunks per warp");
  const int c_begin = part * (NC / NPART), c_end = c_begin + NC / NPART;
  if constexpr (EPI == EPI_SWIGLU) {
    // out0 = act (NULL when only G and U are wanted: backward recompute)
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
      uint32_t g[32], u[32];
      tmem_ld_32(tacc + c, g);
      tmem_ld_32(tacc + BN / 2 + c, u);
      tmem_ld_wait();
      float a[32], gf[32], uf[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        gf[j] = __uint_as_float(g[j]);
        uf[j] = __uint_as_float(u[j]);
        a[j] = silu_f(gf[j]) * uf[j];
      }
      if (p.out0) store_chunk_tma(scratch, nb, lane, &p.to0, tl.n0 + c, yb, a);
      if (p.out1) {
        store_chunk_tma(scratch, nb, lane, &p.to1, tl.n0 + c, yb, gf);
        store_chunk_tma(scratch, nb, lane, &p.to2, tl.n0 + c, yb, uf);
      }
    }
  } else if constexpr (EPI == EPI_STORE && NPART == 4) {
    // one scratch buffer: a chunk per round, the previous store read first
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
      uint32_t r[32];
      tmem_ld_32(tacc + c, r);
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      stage_chunk(scratch, lane, v);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&p.to0, scratch, tl.n0 + c, yb);
        bulk_commit();
      }
    }
  } else if constexpr (EPI == EPI_STORE) {
    // two chunks per round: both TMEM loads under one wait, both buffers
    // under one proxy fence
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 64) {
      uint32_t r0[32], r1[32];
      tmem_ld_32(tacc + c, r0);
      tmem_ld_32(tacc + c + 32, r1);
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r0[j]);
      stage_chunk(scratch, lane, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r1[j]);
      stage_chunk(scratch + kStoreBuf, lane, v);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&p.to0, scratch, tl.n0 + c, yb);
        tma_store_2d(&p.to0, scratch + kStoreBuf, tl.n0 + c + 32, yb);
        bulk_commit();
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU_BWD) {
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
      uint32_t r[32];
      tmem_ld_32(tacc + c, r);
      float gf[32], uf[32], dg[32], du[32];
      // G and U as 64-byte row segments, 4 lanes per row, exchanged through
      // the first scratch buffer once no store still reads it (each element
      // is read here before this warp stores it, so dG, dU may alias G, U)
      uint4 wg[4], wu[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t o = (row_base + 8 * i + (lane >> 2)) * p.ldo + tl.n0 + c + 8 * (lane & 3);
        wg[i] = *reinterpret_cast<const uint4*>(p.aux0 + o);
        wu[i] = *reinterpret_cast<const uint4*>(p.aux1 + o);
      }
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      tmem_ld_wait();
      rows_from_coalesced(scratch, lane, wg, gf);
      rows_from_coalesced(scratch, lane, wu, uf);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float da = __uint_as_float(r[j]);
        const float sig = 1.f / (1.f + expf(-gf[j]));
        dg[j] = da * uf[j] * sig * (1.f + gf[j] * (1.f - sig));
        du[j] = da * gf[j] * sig;
      }
      // both buffers are free: every earlier store was waited for above
      stage_chunk(scratch, lane, dg);
      stage_chunk(scratch + kStoreBuf, lane, du);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&p.to0, scratch, tl.n0 + c, yb);
        tma_store_2d(&p.to1, scratch + kStoreBuf, tl.n0 + c, yb);
        bulk_commit();
      }
    }
  } else if constexpr (EPI == EPI_WGRAD || EPI == EPI_WGRAD_PAIR) {
    const int64_t off = (int64_t)tl.e * p.out_estride + (int64_t)(tl.m0 + row) * p.ldo + tl.n0;
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
      uint32_t r[32];
      tmem_ld_32(tacc + c, r);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      if (scratch) {
        // rows are output rows m0 + row (lane i: m0 + row - lane + i)
        const int64_t o = (int64_t)tl.e * p.out_estride + (int64_t)(tl.m0 + row - lane) * p.ldo + tl.n0;
        if (EPI == EPI_WGRAD_PAIR && c >= BN / 2) store_chunk_coalesced(scratch, lane, p.out1 + o + (c - BN / 2), p.ldo, v);
        else store_chunk_coalesced(scratch, lane, p.out0 + o + c, p.ldo, v);
      } else if (EPI == EPI_WGRAD_PAIR && c >= BN / 2) {
        store_row_bf16x32(p.out1 + off + (c - BN / 2), v);
      } else {
        store_row_bf16x32(p.out0 + off + c, v);
      }
    }
  } else if constexpr (EPI == EPI_ROUTER_DX) {
    // router backward, dense: out0[t, n0 + c] = (D * W_r^T)[t, n0 + c] for the
    // tile's rows below P (= N); the unpermute pass then adds the K rows
    const bool valid = grow < p.P;
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
      uint32_t r[32];
      tmem_ld_32(tacc + c, r);
      tmem_ld_wait();
      if (valid) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        store_row_bf16x32(p.out0 + grow * p.ldo + tl.n0 + c, v);
      }
    }
  }
}

// B tile of one k block into sb; k is the k offset (ROWS / DENSE) or the
// group row (WGRAD); tb is the map to read (SPLIT_K picks it per k block).
// In a pair each CTA fetches its half of B's columns (SPLIT_N: W1 | W3).  On a
// lone unit (an M = 128 pair MMA, see the kernel) CTA r's half feeds the TMEM
// lanes 64r.. of both CTAs, so with SPLIT_N each CTA takes 64 columns of W1
// and the same 64 of W3, keeping a gate and its up projection in one lane.
// slab: bytes between the 64-wide MN slabs of an MN-major B in shared memory
// (8 KB: one 64-deep k block per box; 16 KB: 128-deep boxes, see the kernel).
template <int BN, int CG, int SCHED, bool B_MN, int SPLIT>
__device__ __forceinline__ void load_b(const Params& p, const Tile& tl, uint32_t sb, uint32_t fb,
                                       uint32_t rank, int k, const CUtensorMap* tb, bool lone = false,
                                       uint32_t slab = 8192) {
  if constexpr (CG == 2) {
    if constexpr (SCHED == SCHED_ROWS && B_MN && SPLIT == SPLIT_N && BN == 256) {
      if (lone) {   // one 64-column box of W1 and the same of W3 per CTA
        tma_load_3d_pair(sb, &p.tb0, fb, tl.n0 + 64 * (int)rank, k, tl.e);
        tma_load_3d_pair(sb + slab, &p.tb1, fb, tl.n0 + 64 * (int)rank, k, tl.e);
        return;
      }
    }
    if constexpr (SCHED == SCHED_WGRAD) {
#pragma unroll
      for (int j = 0; j < BN / 128; ++j) {
        if (SPLIT == SPLIT_N)
          tma_load_2d_pair(sb + j * slab, rank ? &p.tb1 : &p.tb0, fb, tl.n0 + 64 * j, k);
        else
          tma_load_2d_pair(sb + j * slab, tb, fb, tl.n0 + (BN / 2) * (int)rank + 64 * j, k);
      }
    } else if constexpr (B_MN) {
#pragma unroll
      for (int j = 0; j < BN / 128; ++j) {
        if (SPLIT == SPLIT_N)
          tma_load_3d_pair(sb + j * slab, rank ? &p.tb1 : &p.tb0, fb, tl.n0 + 64 * j, k, tl.e);
        else
          tma_load_3d_pair(sb + j * slab, tb, fb, tl.n0 + (BN / 2) * (int)rank + 64 * j, k, tl.e);
      }
    } else {
      tma_load_3d_pair(sb, tb, fb, k, tl.n0 + (BN / 2) * (int)rank, tl.e);
    }
  } else {
    if constexpr (SCHED == SCHED_WGRAD) {
#pragma unroll
      for (int j = 0; j < BN / 64; ++j) {
        if (SPLIT == SPLIT_N && j >= BN / 128)
          tma_load_2d(sb + j * 8192, &p.tb1, fb, tl.n0 + 64 * (j - BN / 128), k);
        else
          tma_load_2d(sb + j * 8192, tb, fb, tl.n0 + 64 * j, k);
      }
    } else if constexpr (SCHED == SCHED_DENSE && B_MN) {
      for (int j = 0; j < p.n_mma / 64; ++j) tma_load_2d(sb + j * 8192, tb, fb, 64 * j, k);
    } else if constexpr (SCHED == SCHED_DENSE) {
      tma_load_2d(sb, tb, fb, k, tl.n0);
    } else if constexpr (B_MN) {
#pragma unroll
      for (int j = 0; j < BN / 64; ++j) {
        if (SPLIT == SPLIT_N && j >= BN / 128)
          tma_load_3d(sb + j * 8192, &p.tb1, fb, tl.n0 + 64 * (j - BN / 128), k, tl.e);
        else
          tma_load_3d(sb + j * 8192, tb, fb, tl.n0 + 64 * j, k, tl.e);
      }
    } else {
      tma_load_3d(sb, tb, fb, k, tl.n0, tl.e);
    }
  }
}

template <int BN, int MT, int CG, int SCHED, int EPI, bool A_MN, bool B_MN, int SPLIT, bool GA, int EW>
__global__ void __launch_bounds__(64 + 32 * EW, 1) umma_gemm_kernel(const __grid_constant__ Params p) {
  using S = Shape<BN, MT, CG>;
  constexpr int STAGES = S::STAGES;
  constexpr int STAGE_BYTES = S::STAGE_BYTES;
  constexpr int KSUB = S::KSUB;
  // Stage layout: the A tiles of the stage's KSUB k blocks, then their B
  // tiles.  A K-major operand is one box per k block.  An MN-major operand of
  // a two-k-block stage (CTA pairs) comes as one 128-deep box per 64-wide MN
  // slab, the slab's two k blocks back to back (16 KB slabs, WSLAB apart):
  // half the TMA operations of 64-deep boxes, which the single producer
  // thread issues one by one.
  constexpr bool WIDE = KSUB == 2 && MT == 1;
  constexpr bool A_WIDE = WIDE && A_MN;
  constexpr bool B_WIDE = WIDE && B_MN;
  constexpr uint32_t WSLAB = 2 * 8192;
  constexpr int A_BYTES = S::A_BYTES;
  constexpr int B_BYTES = S::B_BYTES;
  constexpr int A_REG = KSUB * A_BYTES;                 // bytes of a stage's A tiles
  static_assert(!WIDE || (!A_MN && !B_MN) || (A_BYTES == 2 * 8192 && B_BYTES == 2 * 8192),
                "wide boxes: two 64-wide MN slabs per operand");
  constexpr int ACC_BUFS = S::ACC_BUFS;
  constexpr int ACC_COLS = S::ACC_COLS;
  constexpr int UNIT = S::UNIT;
  constexpr bool PAIR = CG == 2;
  // A pair's unit whose second 128-row tile does not exist (an expert with an
  // odd tile count) runs as an M = 128 pair MMA: CTA r multiplies rows
  // 64r .. 64r + 63 of the tile, and each CTA's TMEM receives its 64 rows
  // twice, lanes 0-63 holding output columns [0, BN/2) and lanes 64-127
  // columns [BN/2, BN), both in accumulator columns [0, BN/2).
  constexpr bool LONE = PAIR && MT == 1 && SCHED == SCHED_ROWS &&
                        (EPI != EPI_SWIGLU || (SPLIT == SPLIT_N && B_MN && BN == 256));
  static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte swizzle atoms aligned");
  static_assert(STAGES >= 2, "pipeline needs at least two stages");
  static_assert(MT == 1 || SCHED != SCHED_DENSE, "the router uses single 128-row tiles");
  static_assert(!PAIR || SCHED != SCHED_DENSE, "the router uses single CTAs");
  static_assert(!GA || (SCHED == SCHED_ROWS && !A_MN && SPLIT != SPLIT_K) || (SCHED == SCHED_WGRAD && A_MN),
                "row gathers feed K-major A of ROWS or MN-major A of WGRAD");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t bar_base = base + STAGES * STAGE_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * STAGES + ACC_BUFS + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 2 * ACC_BUFS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + STAGES * STAGE_BYTES + 8 * S::N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int32_t* s_unit_start = reinterpret_cast<int32_t*>(tmem_holder + 4);   // [E + 1]
  // scratch_bytes<EPI>() per epilogue warp, 512-byte aligned (the 64-byte
  // swizzle of the TMA stores repeats every 512 bytes)
  static_assert(EW == kEpiWarps || (EW == 16 && CG == 1 && MT == 2 && EPI == EPI_STORE),
                "16 epilogue warps: single-CTA 256-row plain stores");
  constexpr int kScratch = EW == 16 ? kStoreBuf : scratch_bytes<EPI>();
  const uint32_t store_scratch = (smem_u32(s_unit_start + 260) + 511u) & ~511u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;          // 0 = leader
  const int64_t tile0 = PAIR ? (int64_t)cluster_id_x() : (int64_t)blockIdx.x;
  const int64_t tstep = PAIR ? (int64_t)nclusters_x() : (int64_t)gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int a = 0; a < ACC_BUFS; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), PAIR ? 2 * EW : EW);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    // grouped rows beyond the buffers' P rows are not computed: report it
    if (SCHED != SCHED_DENSE && blockIdx.x == 0 && p.status && p.padded_bins[p.E - 1] > p.P)
      atomicOr(p.status, MOE_DEVERR_ROWS);
    fence_barrier_init();
    fence_proxy_async();
  }
  if (SCHED == SCHED_ROWS && warp == 2) {
    // units per expert = ceil(tiles_e / UNIT); exclusive scan over experts
    int carry = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + lane;
      int u = 0;
      if (e < p.E) {
        const int64_t lo = e ? p.padded_bins[e - 1] : 0;
        int64_t hi = p.padded_bins[e];
        if (hi > p.P) hi = p.P;
        const int64_t tiles = hi > lo ? (hi - lo) / BM : 0;
        u = (int)((tiles + UNIT - 1) / UNIT);
        if (p.single_mode == 1 && tiles == 1) u = 0;
        else if (p.single_mode == 2) u = tiles == 1 ? 1 : 0;
      }
      int incl = u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < p.E) s_unit_start[e] = carry + incl - u;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_unit_start[p.E] = carry;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.ta0);
    tma_prefetch_desc(&p.tb0);
    if (SPLIT != SPLIT_NONE) tma_prefetch_desc(&p.tb1);
    if (SPLIT == SPLIT_K) tma_prefetch_desc(&p.ta1);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), S::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), S::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();   // barriers visible to the peer
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int64_t ntiles = total_tiles<SCHED, BN, UNIT, EPI>(p, s_unit_start);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if constexpr (GA) {
      // A rows gathered from the token matrix: each lane gathers four rows
      // (ROWS: rows 4*lane.. of each 128-row half; WGRAD: k rows 4*(lane%16)..
      // of column box lane/16); lane 0 arms the barrier and loads B
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const int g = lane & 15, jb = lane >> 4;
      for (int64_t t = tile0; t < ntiles && ok; t += tstep) {
        const Tile tl = get_tile<SCHED, BN, UNIT, EPI>(p, t, s_unit_start);
        const int64_t pstart = tl.e ? p.padded_bins[tl.e - 1] : 0;
        const int32_t bstart = tl.e ? p.g_bins[tl.e - 1] : 0;
        const int64_t cnt = (int64_t)p.g_bins[tl.e] - bstart;
        auto tok_of = [&](int64_t r) -> int {
          const int64_t j = r - pstart;
          return j < cnt ? p.g_indices[bstart + j] / p.g_K : p.g_N;
        };
        const int n_mma_h = PAIR ? (tl.halves + 1) / 2 : tl.halves;
        // bytes landing per k block (A, B) and per stage (wide boxes bring
        // both k blocks of a stage whatever nsub is)
        const uint32_t txa = (PAIR ? 2u : 1u) * (uint32_t)((PAIR ? n_mma_h : tl.halves) * BM * BK * 2);
        const uint32_t txb = (PAIR ? 2u : 1u) * (uint32_t)B_BYTES;
        int tk[MT][4];      // ROWS: this lane's four tokens of each half
        int nx[4];          // WGRAD: this lane's four tokens of the next k block
        if constexpr (SCHED == SCHED_ROWS) {
#pragma unroll
          for (int h = 0; h < MT; ++h) {
            const int hh = PAIR ? 2 * h + (int)rank : h;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              tk[h][i] = h < n_mma_h ? tok_of(tl.row0 + (LONE && tl.halves == 1 ? 64 * (int)rank : hh * BM) +
                                              4 * lane + i)
                                     : p.g_N;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) nx[i] = tl.nkb > 0 ? tok_of(tl.row0 + 4 * g + i) : p.g_N;
        }
        for (int kb0 = 0; kb0 < tl.nkb; kb0 += KSUB) {
          const int nsub = (tl.nkb - kb0) < KSUB ? (tl.nkb - kb0) : KSUB;
          int w_ok = 1;
          if (lane == 0)
            w_ok = mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status, kTimeoutNs) ? 1 : 0;
          w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
          if (!w_ok) { ok = false; break; }
          const uint32_t fb = PAIR ? map_to_rank(full_bar(stage), 0) : full_bar(stage);
          // A arrives gathered, k block by k block (nsub of them); a wide B box
          // brings both k blocks of the stage
          if (lane == 0 && (!PAIR || rank == 0))
            mbar_expect_tx(full_bar(stage), txa * (uint32_t)nsub + txb * (uint32_t)(B_WIDE ? KSUB : nsub));
          const uint32_t st0 = base + stage * STAGE_BYTES;
          for (int j = 0; j < nsub; ++j) {
            const int kb = kb0 + j;
            const uint32_t sa = st0 + j * A_BYTES;               // K-major A of k block j
            const uint32_t sb = st0 + A_REG + j * B_BYTES;       // K-major B of k block j
            const int kc = SCHED == SCHED_WGRAD ? (int)(tl.row0 + (int64_t)kb * BK) : kb * BK;
            if (lane == 0) {
              if constexpr (B_WIDE) {
                if (j == 0) load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, st0 + A_REG, fb, rank, kc, &p.tb0,
                                                               LONE && tl.halves == 1, WSLAB);
              } else {
                load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, sb, fb, rank, kc, &p.tb0, LONE && tl.halves == 1);
              }
            }
            if constexpr (SCHED == SCHED_WGRAD) {
              int cur[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) cur[i] = nx[i];
              for (int h = 0; h < n_mma_h; ++h) {
                const int hh = PAIR ? 2 * h + (int)rank : h;
                // MN-major A gathered k row by k row: slab jb, rows 4g.. of k block j
                const uint32_t dst = A_WIDE ? st0 + jb * WSLAB + j * 8192 + g * 512
                                            : sa + h * (BM * BK * 2) + jb * 8192 + g * 512;
                const int m = tl.m0 + BM * hh + 64 * jb;
                if constexpr (PAIR) tma_gather4_pair(dst, &p.ta0, fb, m, cur[0], cur[1], cur[2], cur[3]);
                else tma_gather4(dst, &p.ta0, fb, m, cur[0], cur[1], cur[2], cur[3]);
              }
              if (kb + 1 < tl.nkb) {
#pragma unroll
                for (int i = 0; i < 4; ++i) nx[i] = tok_of((int64_t)kc + BK + 4 * g + i);
              }
            } else {
#pragma unroll
              for (int h = 0; h < MT; ++h) {
                if (h < n_mma_h) {
                  const uint32_t dst = sa + h * (BM * BK * 2) + lane * 512;
                  if constexpr (PAIR) tma_gather4_pair(dst, &p.ta0, fb, kc, tk[h][0], tk[h][1], tk[h][2], tk[h][3]);
                  else tma_gather4(dst, &p.ta0, fb, kc, tk[h][0], tk[h][1], tk[h][2], tk[h][3]);
                }
              }
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {}
      }
    } else if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t t = tile0; t < ntiles && ok; t += tstep) {
        const Tile tl = get_tile<SCHED, BN, UNIT, EPI>(p, t, s_unit_start);
        // MMAs of this tile: with a pair, MMA h covers tiles 2h and 2h+1 of the
        // unit (one per CTA) and runs when tile 2h exists
        const int n_mma_h = PAIR ? (tl.halves + 1) / 2 : tl.halves;
        // bytes landing per k block (A, B; a pair counts both CTAs' loads)
        const uint32_t txa = PAIR ? 2u * (uint32_t)(n_mma_h * BM * BK * 2) : (uint32_t)tl.halves * BM * BK * 2;
        const uint32_t txb = PAIR ? 2u * (uint32_t)B_BYTES
                                  : (SCHED == SCHED_DENSE ? (uint32_t)p.n_mma * BK * 2 : (uint32_t)B_BYTES);
        for (int kb0 = 0; kb0 < tl.nkb; kb0 += KSUB) {
          const int nsub = (tl.nkb - kb0) < KSUB ? (tl.nkb - kb0) : KSUB;
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status, kTimeoutNs)) { ok = false; break; }
          const uint32_t fb = PAIR ? map_to_rank(full_bar(stage), 0) : full_bar(stage);   // the leader's barrier
          if (!PAIR || rank == 0)
            mbar_expect_tx(full_bar(stage), txa * (uint32_t)(A_WIDE ? KSUB : nsub) + txb * (uint32_t)(B_WIDE ? KSUB : nsub));
          const uint32_t st0 = base + stage * STAGE_BYTES;
          for (int j = 0; j < nsub; ++j) {
            const int kb = kb0 + j;
            const uint32_t sa = st0 + j * A_BYTES;               // K-major A of k block j
            const uint32_t sb = st0 + A_REG + j * B_BYTES;       // K-major B of k block j
            if constexpr (PAIR) {
              if constexpr (SCHED == SCHED_WGRAD) {
                const int krow = (int)(tl.row0 + (int64_t)kb * BK);
                if constexpr (A_WIDE) {
                  if (j == 0) {          // both k blocks of the stage, one 128-deep box per slab
                    const int m = tl.m0 + BM * (int)rank;
                    tma_load_2d_pair(st0, &p.ta0, fb, m, krow);
                    tma_load_2d_pair(st0 + WSLAB, &p.ta0, fb, m + 64, krow);
                  }
                } else {
                  for (int h = 0; h < n_mma_h; ++h) {
                    const int m = tl.m0 + BM * (2 * h + (int)rank);
                    tma_load_2d_pair(sa + h * (BM * BK * 2), &p.ta0, fb, m, krow);
                    tma_load_2d_pair(sa + h * (BM * BK * 2) + 8192, &p.ta0, fb, m + 64, krow);
                  }
                }
                if constexpr (B_WIDE) {
                  if (j == 0) load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, st0 + A_REG, fb, rank, krow, &p.tb0, false, WSLAB);
                } else {
                  load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, sb, fb, rank, krow, &p.tb0);
                }
              } else {
                int k = kb * BK;
                const CUtensorMap* ta = &p.ta0;
                const CUtensorMap* tb = &p.tb0;
                if (SPLIT == SPLIT_K && k >= p.ksplit) { k -= p.ksplit; ta = &p.ta1; tb = &p.tb1; }
                const bool lone = LONE && tl.halves == 1;
                for (int h = 0; h < n_mma_h; ++h)
                  tma_load_2d_pair(sa + h * (BM * BK * 2), ta, fb, k,
                                   (int)tl.row0 + (lone ? 64 * (int)rank : BM * (2 * h + (int)rank)));
                if constexpr (B_WIDE) {
                  if (j == 0) load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, st0 + A_REG, fb, rank, k, tb, lone, WSLAB);
                } else {
                  load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, sb, fb, rank, k, tb, lone);
                }
              }
            } else {
              if constexpr (SCHED == SCHED_WGRAD) {
                const int krow = (int)(tl.row0 + (int64_t)kb * BK);
                // A = X^T: 64-wide MN boxes of the [rows, M] matrix, 2 per half
#pragma unroll
                for (int q = 0; q < 2 * MT; ++q) tma_load_2d(sa + q * 8192, &p.ta0, fb, tl.m0 + 64 * q, krow);
                load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, sb, fb, 0u, krow, &p.tb0);
              } else {
                int k = kb * BK;
                const CUtensorMap* ta = &p.ta0;
                const CUtensorMap* tb = &p.tb0;
                if (SPLIT == SPLIT_K && k >= p.ksplit) { k -= p.ksplit; ta = &p.ta1; tb = &p.tb1; }
                tma_load_2d(sa, ta, fb, k, (int)tl.row0);
                if (MT == 2 && tl.halves == 2) tma_load_2d(sa + BM * BK * 2, ta, fb, k, (int)tl.row0 + BM);
                load_b<BN, CG, SCHED, B_MN, SPLIT>(p, tl, sb, fb, 0u, k, tb);
              }
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // give the loads already issued a bounded chance to land
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      const int n_mma = (SCHED == SCHED_DENSE) ? p.n_mma : BN;
      const uint32_t idesc_full = idesc_bf16(PAIR ? 2 * BM : BM, n_mma, A_MN, B_MN);
      const uint32_t idesc_lone = idesc_bf16(BM, n_mma, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t t = tile0; t < ntiles && ok; t += tstep) {
        const Tile tl = get_tile<SCHED, BN, UNIT, EPI>(p, t, s_unit_start);
        if (tl.nkb == 0) continue;
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status, kTimeoutNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        const uint32_t idesc = (LONE && tl.halves == 1) ? idesc_lone : idesc_full;
        for (int kb0 = 0; kb0 < tl.nkb; kb0 += KSUB) {
          const int nsub = (tl.nkb - kb0) < KSUB ? (tl.nkb - kb0) : KSUB;
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status, kTimeoutNs)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < KSUB; ++j) {
            if (j < nsub) {
              const uint32_t st0 = base + stage * STAGE_BYTES;
              const uint32_t sa = st0 + j * A_BYTES;
              const uint32_t sb = st0 + A_REG + j * B_BYTES;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                const uint64_t bd = B_WIDE ? desc_mn_sw128(st0 + A_REG + j * 8192 + kk * 2048, WSLAB)
                                           : (B_MN ? desc_mn_sw128(sb + kk * 2048, 8192) : desc_k_sw128(sb + kk * 32));
                const uint32_t accum = ((kb0 + j) | kk) != 0 ? 1u : 0u;
                if constexpr (PAIR) {
#pragma unroll
                  for (int h = 0; h < MT; ++h) {
                    if (2 * h < tl.halves) {
                      const uint32_t ah = sa + h * (BM * BK * 2);
                      const uint64_t ad = A_WIDE ? desc_mn_sw128(st0 + j * 8192 + kk * 2048, WSLAB)
                                                 : (A_MN ? desc_mn_sw128(ah + kk * 2048, 8192) : desc_k_sw128(ah + kk * 32));
                      mma_bf16_pair(d_tmem + h * BN, ad, bd, idesc, accum);
                    }
                  }
                } else {
#pragma unroll
                  for (int h = 0; h < MT; ++h) {
                    if (h < tl.halves) {
                      const uint32_t ah = sa + h * (BM * BK * 2);
                      const uint64_t ad = A_MN ? desc_mn_sw128(ah + kk * 2048, 8192) : desc_k_sw128(ah + kk * 32);
                      mma_bf16(d_tmem + h * BN, ad, bd, idesc, accum);
                    }
                  }
                }
              }
            }
          }
          // smem slot free (in both CTAs of a pair) once these MMAs are done
          if constexpr (PAIR) mma_commit_pair(empty_bar(stage), 0x3); else mma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        // accumulator ready for the epilogue(s)
        if constexpr (PAIR) mma_commit_pair(tfull_bar(acc), 0x3); else mma_commit(tfull_bar(acc));
        if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        if constexpr (PAIR) mma_commit_pair(drain_bar, 0x1); else mma_commit(drain_bar);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer() - t0 < 50000000ull) {}
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                       // TMEM lane quarter of this warp
    const int part = (warp - 2) >> 2;             // which half of the columns
    const int row = q * 32 + lane;                // row inside a 128-row half
    const uint32_t tempty_leader0 = PAIR ? map_to_rank(tempty_bar(0), 0) : 0u;
    int nb = 0;                                   // next TMA-store scratch buffer
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t t = tile0; t < ntiles; t += tstep) {
      const Tile tl = get_tile<SCHED, BN, UNIT, EPI>(p, t, s_unit_start);
      if constexpr (SCHED == SCHED_WGRAD) {
        if (tl.nkb == 0) {                        // expert with no rows: zero gradient
          const float z[32] = {0.f};
#pragma unroll 1
          for (int h = 0; h < MT; ++h) {
            const int hh = PAIR ? 2 * h + (int)rank : h;
            const int64_t off = (int64_t)tl.e * p.out_estride + (int64_t)(tl.m0 + hh * BM + row) * p.ldo + tl.n0;
            if constexpr (EPI == EPI_WGRAD_PAIR) {
#pragma unroll 1
              for (int c = part * (BN / 4); c < (part + 1) * (BN / 4); c += 32) {
                store_row_bf16x32(p.out0 + off + c, z);
                store_row_bf16x32(p.out1 + off + c, z);
              }
            } else {
#pragma unroll 1
              for (int c = part * (BN / 2); c < (part + 1) * (BN / 2); c += 32) store_row_bf16x32(p.out0 + off + c, z);
            }
          }
          continue;
        }
      }
      int ok = 0;
      // a wait that spans the tile's main loop: sleep between polls (measured
      // 1-2.5 % faster per GEMM in the power-capped step: the clock gains
      // more than the up to 256 ns a late wake-up costs)
      if (lane == 0) ok = mbar_wait_bounded_sleep(tfull_bar(acc), acc_phase, abort_flag, p.status, kTimeoutNs) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      bool lone_done = false;
      if constexpr (LONE) {
        if (tl.halves == 1) {
          // M = 128 result: rows 64 * rank + (q & 1) * 32 + lane, lanes 64g..
          // holding output columns [g * BN/2, (g + 1) * BN/2) of the MMA (with
          // SPLIT_N SwiGLU: 64 gate and 64 up columns of act columns 64g..)
          const int g = q >> 1;
          const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
          Tile th = tl;
          th.row0 = tl.row0 + 64 * (int)rank;
          th.n0 = tl.n0 + g * (EPI == EPI_SWIGLU ? BN / 4 : BN / 2);
          epilogue_half<BN / 2, SCHED, EPI>(p, th, tacc, (q & 1) * 32 + lane, part,
                                            kScratch ? store_scratch + (warp - 2) * kScratch : 0u, nb);
          lone_done = true;
        }
      }
      if constexpr (PAIR) {
        // this CTA's tiles 2h + rank of the unit; tiles past the expert's end
        // (a short last unit) are computed on garbage rows and not stored
#pragma unroll 1
        for (int h = 0; h < MT && !lone_done; ++h) {
          const int j = 2 * h + (int)rank;
          if (j >= tl.halves) continue;
          const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS + h * BN);
          Tile th = tl;
          if (SCHED == SCHED_WGRAD) th.m0 = tl.m0 + j * BM; else th.row0 = tl.row0 + j * BM;
          epilogue_half<BN, SCHED, EPI>(p, th, tacc, row, part,
                                        kScratch ? store_scratch + (warp - 2) * kScratch : 0u, nb);
        }
      } else {
#pragma unroll 1
        for (int h = 0; h < tl.halves; ++h) {
          const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS + h * BN);
          Tile th = tl;
          if (SCHED == SCHED_WGRAD) th.m0 = tl.m0 + h * BM; else th.row0 = tl.row0 + h * BM;
          epilogue_half<BN, SCHED, EPI, EW / 4>(p, th, tacc, row, part,
                                        kScratch ? store_scratch + (warp - 2) * kScratch : 0u, nb);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_remote(tempty_leader0 + 8u * acc);   // the leader's barrier
        else mbar_arrive(tempty_bar(acc));
      }
      if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
    }
    // the TMA stores have read their scratch and written global memory
    if (store_mode<EPI>() == STORE_TMA && lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
    else tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

// 2-D bf16 map over a row-major [outer, inner] matrix, 128-byte swizzle.
static bool map2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_elems,
                  uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;

  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map over a row-major [outer, inner] output for TMA stores of
// 32 x 32 chunks, 64-byte swizzle (one 64-byte chunk row per swizzle row).
static bool map_out2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_elems) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_elems * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over [d2, d1, d0] (d0 contiguous), 128-byte swizzle, box depth 1.
static bool map3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint32_t box0, uint32_t box1) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

template <int BN, int MT, int CG, int SCHED, int EPI, bool A_MN, bool B_MN, int SPLIT, bool GA = false,
          int EW = kEpiWarps>
static moe_status launch(const char* name, const Params& p_in, int64_t tiles_upper, cudaStream_t s) {
  using S = Shape<BN, MT, CG>;
  Params p = p_in;
  if (p.group_m <= 0) p.group_m = kGroupM;
  auto kern = umma_gemm_kernel<BN, MT, CG, SCHED, EPI, A_MN, B_MN, SPLIT, GA, EW>;
  constexpr size_t per_warp = EW == 16 ? kStoreBuf : scratch_bytes<EPI>();
  constexpr size_t scratch = per_warp ? (size_t)EW * per_warp + 512 : 0;
  static_assert(S::SMEM + scratch <= 232448, "shared memory per CTA");
  const size_t smem = S::SMEM + scratch;
  // once per device: later calls (a CUDA graph capture among them) only launch
  static bool smem_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!smem_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
      (void)cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    smem_set[dev] = true;
  }
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.blockDim = dim3(64 + 32 * EW, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Persistent CTAs (or pairs): every one must be resident at once, since each
  // owns a fixed share of the tiles.  Pairs are placed within a GPC, so ask the
  // runtime how many fit rather than assuming SMs / 2.
  int64_t units = sm_count();
  if (CG == 2) {
    static int cached[64] = {0};
    if (!cached[dev]) {
      int n = 0;
      cfg.gridDim = dim3((unsigned)sm_count(), 1, 1);
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        n = sm_count() / 2;
      }
      cached[dev] = n;
    }
    units = cached[dev];
  }
  int64_t grid = tiles_upper < units ? tiles_upper : units;
  if (grid < 1) grid = 1;
  cfg.gridDim = dim3((unsigned)(grid * CG), 1, 1);
  cudaError_t err = cudaSuccess;
  MOE_TRACED(name, s, (err = cudaLaunchKernelEx(&cfg, kern, p)));
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

static void set_gather(Params* p, const RowGather* ga) {
  p->g_indices = ga->indices;
  p->g_bins = ga->bins;
  p->g_K = ga->K;
  p->g_N = ga->N;
}

static Params blank_params(const int32_t* pb, int E, int64_t P, int* status) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.padded_bins = pb;
  p.E = E;
  p.P = P;
  p.status = status;
  return p;
}

}  // namespace umma

using namespace umma;

bool umma_shape_supported(int H, int F) { return H % 128 == 0 && F % 128 == 0 && H >= 128 && F >= 128; }

// Kernel choice per GEMM (measured on B200, interleaved in one process on the
// training-step and forward workloads).  A CTA pair (256 x 256, one 128-row
// tile per CTA) halves each CTA's B traffic and keeps two accumulator sets in
// TMEM, so a heavy epilogue (SwiGLU, SwiGLU backward, weight gradients)
// overlaps the next tile's main loop; but a pair always multiplies 256 rows,
// and an expert with an odd tile count wastes half of its last unit.  A single
// CTA with two 128-row halves (256 x 256, one accumulator set) skips the MMA of
// a missing half; with a light store epilogue that wins: GEMM2 and the dgrad
// to x run that way (GEMM2 8-20 % faster than in pairs), the rest in pairs.

// [G | U] = x_perm * [W1_e | W3_e] per group; act = silu(G) * U.  act, G and U
// may each be NULL (the backward's recompute asks for G and U only).
moe_status gemm1_umma(const void* x_perm, const void* W1, const void* W3, const int32_t* pb, int E, int H,
                      int F, int64_t P, void* act, void* G, void* U, int* status, cudaStream_t s,
                      const char* name, const RowGather* ga) {
  typedef __nv_bfloat16 bf;
  Params p = blank_params(pb, E, P, status);
  const bool a_ok = ga ? map2d(&p.ta0, ga->x, H, ga->N, H, 64, 1) : map2d(&p.ta0, x_perm, H, P, H, 64, 128);
  // CTA pairs read MN-major operands in 128-deep boxes (two k blocks, see the kernel)
  if (!a_ok || !map3d(&p.tb0, W1, F, H, E, 64, 128) || !map3d(&p.tb1, W3, F, H, E, 64, 128))
    return MOE_ERR_CUDA;
  if (ga) set_gather(&p, ga);
  if ((act && !map_out2d(&p.to0, act, F, P, F)) || (G && !map_out2d(&p.to1, G, F, P, F)) ||
      (U && !map_out2d(&p.to2, U, F, P, F)))
    return MOE_ERR_CUDA;
  p.kdim = H;
  p.n_mma = 256;
  p.n_tiles = F / 128;
  p.out0 = (bf*)act;
  p.out1 = (bf*)G;
  p.out2 = (bf*)U;
  p.ldo = F;
  const int64_t up = (P / BM) * p.n_tiles;
  if (ga) return launch<256, 1, 2, SCHED_ROWS, EPI_SWIGLU, false, true, SPLIT_N, true>(name, p, up, s);
  // Many experts of a single 128-row tile (row buffer of at most 4 tiles per
  // expert on average: fine-grained layers): a pair would run each of them as
  // a lone unit, which costs about as much as a full one, so they go to a
  // second, single-CTA launch (M = 128 per SM, no rows idle) and the pairs
  // take the experts of two or more tiles.
  if (P <= (int64_t)E * 4 * BM) {
    p.single_mode = 1;
    moe_status st = launch<256, 1, 2, SCHED_ROWS, EPI_SWIGLU, false, true, SPLIT_N>(name, p, up, s);
    if (st != MOE_OK) return st;
    Params q = p;
    q.single_mode = 2;
    // single-CTA stages hold one k block: 64-deep weight boxes
    if (!map3d(&q.tb0, W1, F, H, E, 64, 64) || !map3d(&q.tb1, W3, F, H, E, 64, 64)) return MOE_ERR_CUDA;
    const int64_t uq = (int64_t)E * q.n_tiles;
    return launch<256, 1, 1, SCHED_ROWS, EPI_SWIGLU, false, true, SPLIT_N>("gemm1_swiglu_single", q, uq, s);
  }
  return launch<256, 1, 2, SCHED_ROWS, EPI_SWIGLU, false, true, SPLIT_N>(name, p, up, s);
}

moe_status grouped_swiglu_umma(const void* x_perm, const void* W1, const void* W3, const void* W2,
                               const int32_t* pb, int E, int H, int F, int64_t P, void* act, void* out,
                               void* gate_up, int* status, cudaStream_t s, const RowGather* ga) {
  typedef __nv_bfloat16 bf;
  // GEMM1 + SwiGLU: [G | U] = x_perm * [W1_e | W3_e], act = silu(G) * U
  moe_status st = gemm1_umma(x_perm, W1, W3, pb, E, H, F, P, act,
                             gate_up ? (bf*)gate_up : nullptr,
                             gate_up ? (bf*)gate_up + (size_t)P * F : nullptr, status, s, "gemm1_swiglu", ga);
  if (st != MOE_OK) return st;
  // GEMM2: out = act * W2_e
  {
    Params p = blank_params(pb, E, P, status);
    const int bn = (H % 256 == 0) ? 256 : 128;
    if (!map2d(&p.ta0, act, F, P, F, 64, 128) || !map3d(&p.tb0, W2, H, F, E, 64, 64) ||
        !map_out2d(&p.to0, out, H, P, H))
      return MOE_ERR_CUDA;
    p.kdim = F;
    p.n_mma = bn;
    p.n_tiles = H / bn;
    p.out0 = (bf*)out;
    p.ldo = H;
    const int64_t up = (P / BM) * p.n_tiles;
    if (bn == 256) return launch<256, 2, 1, SCHED_ROWS, EPI_STORE, false, true, SPLIT_NONE, false, 16>("gemm2", p, up, s);
    return launch<128, 1, 1, SCHED_ROWS, EPI_STORE, false, true, SPLIT_NONE>("gemm2", p, up, s);
  }
}

moe_status grouped_swiglu_bwd_umma(const void* d_out, const void* x_perm, const void* act,
                                   const void* gate_up, const void* W1, const void* W3, const void* W2,
                                   const int32_t* pb, int E, int H, int F, int64_t P, void* d_gate_up,
                                   void* dW1, void* dW3, void* dW2, void* dx_perm, int* status,
                                   cudaStream_t s, const RowGather* ga) {
  typedef __nv_bfloat16 bf;
  const bf* G = (const bf*)gate_up;
  const bf* U = G + (size_t)P * F;
  bf* dG = (bf*)d_gate_up;
  bf* dU = dG + (size_t)P * F;
  const bool pref = true;
  moe_status st;
  // dA = d_out * W2_e^T with the SwiGLU backward in the epilogue
  {
    Params p = blank_params(pb, E, P, status);
    const int bn = (F % 256 == 0) ? 256 : 128;
    const bool pair = pref && bn == 256;
    if (!map2d(&p.ta0, d_out, H, P, H, 64, 128) || !map3d(&p.tb0, W2, H, F, E, 64, pair ? bn / 2 : bn) ||
        !map_out2d(&p.to0, dG, F, P, F) || !map_out2d(&p.to1, dU, F, P, F))
      return MOE_ERR_CUDA;
    p.kdim = H;
    p.n_mma = bn;
    p.n_tiles = F / bn;
    p.aux0 = G;
    p.aux1 = U;
    p.out0 = dG;
    p.out1 = dU;
    p.ldo = F;
    const int64_t up = (P / BM) * p.n_tiles;
    // as in GEMM1: with many one-tile experts those run on single CTAs
    const bool split = pair && P <= (int64_t)E * 4 * BM;
    if (split) p.single_mode = 1;
    st = pair ? launch<256, 1, 2, SCHED_ROWS, EPI_SWIGLU_BWD, false, false, SPLIT_NONE>("dgrad_w2_swiglu_bwd", p, up, s)
         : bn == 256 ? launch<256, 1, 1, SCHED_ROWS, EPI_SWIGLU_BWD, false, false, SPLIT_NONE>("dgrad_w2_swiglu_bwd", p, up, s)
                     : launch<128, 1, 1, SCHED_ROWS, EPI_SWIGLU_BWD, false, false, SPLIT_NONE>("dgrad_w2_swiglu_bwd", p, up, s);
    if (st != MOE_OK) return st;
    if (split) {
      Params q = p;
      q.single_mode = 2;
      if (!map3d(&q.tb0, W2, H, F, E, 64, bn)) return MOE_ERR_CUDA;   // a single CTA reads all BN rows
      st = launch<256, 1, 1, SCHED_ROWS, EPI_SWIGLU_BWD, false, false, SPLIT_NONE>("dgrad_w2_swiglu_bwd_single", q,
                                                                                 (int64_t)E * q.n_tiles, s);
      if (st != MOE_OK) return st;
    }
  }
  // dW2_e = act_e^T * d_out_e   [F, H]
  {
    Params p = blank_params(pb, E, P, status);
    const int bn = (H % 256 == 0) ? 256 : 128;
    const int unit = (bn == 256 && F % 256 == 0) ? 2 : 1;
    const uint32_t kbox = unit == 2 && pref ? 128 : 64;   // CTA pairs: 128-deep MN-major boxes
    if (!map2d(&p.ta0, act, F, P, F, 64, kbox) || !map2d(&p.tb0, d_out, H, P, H, 64, kbox)) return MOE_ERR_CUDA;
    p.n_mma = bn;
    p.m_tiles_w = F / (BM * unit);
    p.n_tiles = H / bn;
    p.out0 = (bf*)dW2;
    p.ldo = H;
    p.out_estride = (int64_t)F * H;
    const int64_t tiles = (int64_t)E * p.m_tiles_w * p.n_tiles;
    if (unit == 2 && pref) st = launch<256, 1, 2, SCHED_WGRAD, EPI_WGRAD, true, true, SPLIT_NONE>("wgrad_w2", p, tiles, s);
    else if (unit == 2) st = launch<256, 2, 1, SCHED_WGRAD, EPI_WGRAD, true, true, SPLIT_NONE>("wgrad_w2", p, tiles, s);
    else if (bn == 256) st = launch<256, 1, 1, SCHED_WGRAD, EPI_WGRAD, true, true, SPLIT_NONE>("wgrad_w2", p, tiles, s);
    else st = launch<128, 1, 1, SCHED_WGRAD, EPI_WGRAD, true, true, SPLIT_NONE>("wgrad_w2", p, tiles, s);
    if (st != MOE_OK) return st;
  }
  // dW1_e | dW3_e = x_perm_e^T * [dG_e | dU_e]   [H, F] each
  {
    Params p = blank_params(pb, E, P, status);
    const int unit = (H % 256 == 0) ? 2 : 1;
    const uint32_t kbox = unit == 2 && (pref || ga) ? 128 : 64;   // CTA pairs: 128-deep MN-major boxes
    const bool a_ok = ga ? map2d(&p.ta0, ga->x, H, ga->N, H, 64, 1) : map2d(&p.ta0, x_perm, H, P, H, 64, kbox);
    if (!a_ok || !map2d(&p.tb0, dG, F, P, F, 64, kbox) || !map2d(&p.tb1, dU, F, P, F, 64, kbox))
      return MOE_ERR_CUDA;
    if (ga) set_gather(&p, ga);
    p.n_mma = 256;
    p.m_tiles_w = H / (BM * unit);
    p.n_tiles = F / 128;
    p.out0 = (bf*)dW1;
    p.out1 = (bf*)dW3;
    p.ldo = F;
    p.out_estride = (int64_t)H * F;
    const int64_t tiles = (int64_t)E * p.m_tiles_w * p.n_tiles;
    if (ga && unit == 2) st = launch<256, 1, 2, SCHED_WGRAD, EPI_WGRAD_PAIR, true, true, SPLIT_N, true>("wgrad_w1_w3", p, tiles, s);
    else if (ga) st = launch<256, 1, 1, SCHED_WGRAD, EPI_WGRAD_PAIR, true, true, SPLIT_N, true>("wgrad_w1_w3", p, tiles, s);
    else if (unit == 2 && pref) st = launch<256, 1, 2, SCHED_WGRAD, EPI_WGRAD_PAIR, true, true, SPLIT_N>("wgrad_w1_w3", p, tiles, s);
    else if (unit == 2) st = launch<256, 2, 1, SCHED_WGRAD, EPI_WGRAD_PAIR, true, true, SPLIT_N>("wgrad_w1_w3", p, tiles, s);
    else st = launch<256, 1, 1, SCHED_WGRAD, EPI_WGRAD_PAIR, true, true, SPLIT_N>("wgrad_w1_w3", p, tiles, s);
    if (st != MOE_OK) return st;
  }
  // dx_perm = dG * W1_e^T + dU * W3_e^T  (one K = 2F contraction)
  {
    Params p = blank_params(pb, E, P, status);
    const int bn = (H % 256 == 0) ? 256 : 128;
    const bool pair = false;    // see the kernel choice note above
    const uint32_t box = pair ? bn / 2 : bn;
    if (!map2d(&p.ta0, dG, F, P, F, 64, 128) || !map2d(&p.ta1, dU, F, P, F, 64, 128) ||
        !map3d(&p.tb0, W1, F, H, E, 64, box) || !map3d(&p.tb1, W3, F, H, E, 64, box) ||
        !map_out2d(&p.to0, dx_perm, H, P, H))
      return MOE_ERR_CUDA;
    p.kdim = 2 * F;
    p.ksplit = F;
    p.n_mma = bn;
    p.n_tiles = H / bn;
    p.out0 = (bf*)dx_perm;
    p.ldo = H;
    const int64_t up = (P / BM) * p.n_tiles;
    st = pair ? launch<256, 1, 2, SCHED_ROWS, EPI_STORE, false, false, SPLIT_K>("dgrad_x", p, up, s)
         : bn == 256 ? launch<256, 2, 1, SCHED_ROWS, EPI_STORE, false, false, SPLIT_K, false, 16>("dgrad_x", p, up, s)
                     : launch<128, 1, 1, SCHED_ROWS, EPI_STORE, false, false, SPLIT_K>("dgrad_x", p, up, s);
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

// ---- dense router backward on tensor cores ----------------------------------

bool router_bwd_umma_supported(int H, int E) { return E % 64 == 0 && E <= 256 && H % 256 == 0; }

// dx = D * W_r^T (the unpermute pass adds the K expert rows afterwards, in
// place): D [N, E] bf16 is K-major A, W_r [H, E] K-major B (its rows are the
// output columns); 128-token x 256-column tiles, K = E.
moe_status router_dx_umma(const void* D, const void* W_r, int N, int H, int E, void* dx, int* status,
                          cudaStream_t s) {
  typedef __nv_bfloat16 bf;
  Params p = blank_params(nullptr, 1, N, status);
  if (!map2d(&p.ta0, D, E, N, E, 64, 128) || !map2d(&p.tb0, W_r, E, H, E, 64, 256)) return MOE_ERR_CUDA;
  p.kdim = E;
  p.n_mma = 256;
  p.n_tiles = H / 256;
  p.out0 = (bf*)dx;
  p.ldo = H;
  return launch<256, 1, 1, SCHED_DENSE, EPI_ROUTER_DX, false, false, SPLIT_NONE>(
      "dense_router_dx", p, cdiv(N, BM) * p.n_tiles, s);
}

}  // namespace moe
