// The Mamba layer's two projections on tcgen05 tensor cores:
//   in_proj   [x | z] = hidden . in_proj_w^T    (M = tokens, N = 2 d_inner, K = d_model)
//   out_proj  out     = y . out_proj_w^T        (M = tokens, N = d_model,   K = d_inner)
// (TransformerLens "Jamba" adapter page, "Architecture overview": in_proj /
// conv1d / x_proj / dt_proj / out_proj.)
//
// C[M, N] = A[M, K] . B[N, K]^T, bf16 operands (row-major, K contiguous), fp32
// accumulation in TMEM, bf16 results.  Columns [0, n_split) go to C0 and
// [n_split, N) to C1, each row-major with its own width, so that in_proj writes
// x and z as the two [tokens, d_inner] matrices the mixer reads.
//
// Persistent kernel, one CTA per SM, 192 threads:
//   warp 0   TMA producer: per 64-wide K chunk, an A tile [128 x 64] and a B
//            tile [256 x 64] (128-byte swizzle) into a ring of kGStages stages;
//   warp 1   TMEM owner and MMA issuer: 4 x tcgen05.mma (M 128, N 256, K 16)
//            per chunk into one of two 256-column accumulators;
//   warps 2-5 epilogue: TMEM -> registers -> bf16 -> global, one tile row per
//            thread, while warp 1 already accumulates the next tile into the
//            other accumulator.
// Tiles are taken in groups of kGroupM row tiles (all column tiles of a group
// before the next group), so the CTAs working at the same time share a compact
// block of A and B in L2.
#include <cuda.h>

#include "jmix_internal.cuh"
#include "sm100.cuh"

namespace jmix {
namespace {

using namespace sm100;

constexpr int kGM = 128;          // tile rows (tokens)
constexpr int kGN = 256;          // tile columns
constexpr int kGK = 64;           // K chunk: one 128-byte swizzle atom of bf16
constexpr int kGStages = 4;
constexpr int kGroupM = 16;       // row tiles per raster group
constexpr int kGThreads = 192;
constexpr int kGABytes = kGM * kGK * 2;                 // 16 KB
constexpr int kGBBytes = kGN * kGK * 2;                 // 32 KB
constexpr int kGStageBytes = kGABytes + kGBBytes;       // 48 KB
constexpr int kGSmem = 1024 + kGStages * kGStageBytes + 256;
constexpr uint32_t kGTmemCols = 512;                    // two accumulators of 256 columns

struct GemmArgs {
  int64_t M, N, K;
  int64_t n_split;     // columns [0, n_split) -> C0, the rest -> C1
  __nv_bfloat16* C0;   // [M, n_split]
  __nv_bfloat16* C1;   // [M, N - n_split] (unused when n_split == N)
  int64_t m_tiles, n_tiles;
  ErrFlags* err;
  const ErrFlags* fold;  // flags of an earlier kernel to carry into err, or null
};

__device__ __forceinline__ void tile_coords(const GemmArgs& g, int64_t t, int64_t& mt,
                                            int64_t& nt) {
  const int64_t per_group = (int64_t)kGroupM * g.n_tiles;
  const int64_t grp = t / per_group, idx = t - grp * per_group;
  const int64_t rows = min((int64_t)kGroupM, g.m_tiles - grp * kGroupM);  // last group may be short
  mt = grp * kGroupM + idx % rows;
  nt = idx / rows;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kGThreads, 1)
    k_gemm_bf16(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
  uint64_t* full = bars;                       // [stages] A and B tiles landed
  uint64_t* empty = bars + kGStages;           // [stages] MMAs done reading the stage
  uint64_t* acc_full = bars + 2 * kGStages;    // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;          // [2] epilogue done reading (4 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_tiles_total = g.m_tiles * g.n_tiles;
  const int kchunks = (int)((g.K + kGK - 1) / kGK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kGTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();   // A may come from the kernel before this one (out_proj reads y)
  if (g.fold && blockIdx.x == 0 && threadIdx.x == 0) {
    if (g.fold->timeout && atomicExch(&g.err->timeout, 1u) == 0u) g.err->where = g.fold->where;
    if (g.fold->bad_input) atomicExch(&g.err->bad_input, 1u);
  }

  if (warp == 0) {
    if (lane == 0) {
      int64_t it = 0;  // K chunks issued by this CTA (ring position)
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < n_tiles_total; t += gridDim.x) {
        int64_t mt, nt;
        tile_coords(g, t, mt, nt);
        for (int kc = 0; kc < kchunks; ++kc, ++it) {
          const int s = (int)(it % kGStages);
          if (it >= kGStages &&
              !mbar_wait(smem_u32(&empty[s]), (uint32_t)((it / kGStages) - 1) & 1u, g.err, 61)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kGStageBytes;
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, (uint32_t)kGStageBytes);
          tma_load_2d(smem_u32(st), &tm_a, fb, kc * kGK, (int32_t)(mt * kGM));
          tma_load_2d(smem_u32(st + kGABytes), &tm_b, fb, kc * kGK, (int32_t)(nt * kGN));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kGM, kGN);
      int64_t it = 0, j = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < n_tiles_total; t += gridDim.x, ++j) {
        const int b = (int)(j & 1);
        if (j >= 2 &&
            !mbar_wait(smem_u32(&acc_empty[b]), (uint32_t)((j >> 1) - 1) & 1u, g.err, 62))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * kGN);
        for (int kc = 0; kc < kchunks; ++kc, ++it) {
          const int s = (int)(it % kGStages);
          if (!mbar_wait(smem_u32(&full[s]), (uint32_t)(it / kGStages) & 1u, g.err, 63)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ab = smem_u32(smem + s * kGStageBytes), bb = ab + kGABytes;
#pragma unroll
          for (int kk = 0; kk < kGK / 16; ++kk)
            umma_f16(d_tmem, sw128_kmajor_desc(ab + kk * 32), sw128_kmajor_desc(bb + kk * 32),
                     idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&empty[s]));
        }
        if (ok) umma_commit(smem_u32(&acc_full[b]));
      }
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 = tile rows
    const int lg = warp & 3;
    int64_t j = 0;
    for (int64_t t = blockIdx.x; t < n_tiles_total; t += gridDim.x, ++j) {
      int64_t mt, nt;
      tile_coords(g, t, mt, nt);
      const int b = (int)(j & 1);
      if (!mbar_wait(smem_u32(&acc_full[b]), (uint32_t)(j >> 1) & 1u, g.err, 64)) break;
      tc_fence_after();
      const int64_t row = mt * kGM + lg * 32 + lane;
      const int64_t n0 = nt * kGN;
      const uint32_t tbase = tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(b * kGN);
#pragma unroll 1
      for (int c = 0; c < kGN; c += 32) {
        uint32_t r[32];
        tmem_ld16(tbase + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(r));
        tmem_ld16(tbase + (uint32_t)(c + 16), *reinterpret_cast<uint32_t(*)[16]>(r + 16));
        tmem_ld_wait();
        if (row < g.M) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // 8 columns = 16 bytes per store
            const int64_t col = n0 + c + 8 * q;
            if (col + 8 > g.N) break;
            const uint4 v = make_uint4(
                pack_bf16x2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
            __nv_bfloat16* dst = col < g.n_split
                                     ? g.C0 + row * g.n_split + col
                                     : g.C1 + row * (g.N - g.n_split) + (col - g.n_split);
            *reinterpret_cast<uint4*>(dst) = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGTmemCols);
  }
}

// ------------------------------------------------------------ CTA-pair form
// The same GEMM with a 256 x 256 tile per CTA pair (cluster of 2): each CTA
// loads half of the tile's A rows and half of its B rows (32 KB per K chunk
// instead of 48 KB for a 128 x 256 tile), the leader issues
// tcgen05.mma.cta_group::2 (M 256, N 256, K 16) over both CTAs' stages, and each
// CTA's TMEM receives its 128 rows.  Barriers: the leader's full[s] counts both
// CTAs' TMA bytes; the leader's commits arrive on empty[s] and acc_full[b] in
// both CTAs; both CTAs' epilogue warps arrive on the leader's acc_empty[b].
constexpr int kPStages = 6;
constexpr int kPHalf = 128;                              // rows of A and of B per CTA
constexpr int kPStageBytes = 2 * kPHalf * kGK * 2;      // 32 KB: A half + B half
constexpr int kPSmem = 1024 + kPStages * kPStageBytes + 256;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    k_gemm_bf16_pair(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPStages * kPStageBytes);
  uint64_t* full = bars;                       // [stages] (leader) both halves landed
  uint64_t* empty = bars + kPStages;           // [stages] the pair MMAs read the stage
  uint64_t* acc_full = bars + 2 * kPStages;    // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;          // [2] (leader) both epilogues done (8 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  // tiles of 256 rows x 256 columns; g.m_tiles counts 256-row tiles here
  const int64_t n_tiles_total = g.m_tiles * g.n_tiles;
  const int kchunks = (int)((g.K + kGK - 1) / kGK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 8);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kGTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();
  if (g.fold && blockIdx.x == 0 && threadIdx.x == 0) {
    if (g.fold->timeout && atomicExch(&g.err->timeout, 1u) == 0u) g.err->where = g.fold->where;
    if (g.fold->bad_input) atomicExch(&g.err->bad_input, 1u);
  }

  if (warp == 0) {
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      for (int64_t t = pair; ok && t < n_tiles_total; t += npairs) {
        int64_t mt, nt;
        tile_coords(g, t, mt, nt);
        for (int kc = 0; kc < kchunks; ++kc, ++it) {
          const int s = (int)(it % kPStages);
          if (it >= kPStages &&
              !mbar_wait(smem_u32(&empty[s]), (uint32_t)((it / kPStages) - 1) & 1u, g.err, 71)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPStageBytes;
          const uint32_t fb = leader_addr(smem_u32(&full[s]));
          // the leader expects both CTAs' bytes on its barrier
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), (uint32_t)(2 * kPStageBytes));
          tma_load_2d_pair(smem_u32(st), &tm_a, fb, kc * kGK,
                           (int32_t)(mt * (2 * kPHalf) + rank * kPHalf));
          tma_load_2d_pair(smem_u32(st + kPHalf * kGK * 2), &tm_b, fb, kc * kGK,
                           (int32_t)(nt * kGN + rank * kPHalf));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_bf16_f32(2 * kPHalf, kGN);
      int64_t it = 0, j = 0;
      bool ok = true;
      for (int64_t t = pair; ok && t < n_tiles_total; t += npairs, ++j) {
        const int b = (int)(j & 1);
        if (j >= 2 &&
            !mbar_wait(smem_u32(&acc_empty[b]), (uint32_t)((j >> 1) - 1) & 1u, g.err, 72))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * kGN);
        for (int kc = 0; kc < kchunks; ++kc, ++it) {
          const int s = (int)(it % kPStages);
          if (!mbar_wait(smem_u32(&full[s]), (uint32_t)(it / kPStages) & 1u, g.err, 73)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ab = smem_u32(smem + s * kPStageBytes), bb = ab + kPHalf * kGK * 2;
#pragma unroll
          for (int kk = 0; kk < kGK / 16; ++kk)
            umma_f16_pair(d_tmem, sw128_kmajor_desc(ab + kk * 32), sw128_kmajor_desc(bb + kk * 32),
                          idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(smem_u32(&empty[s]), 0x3);
        }
        if (ok) umma_commit_pair(smem_u32(&acc_full[b]), 0x3);
      }
    }
  } else {
    // epilogue: this CTA's 128 rows of the pair's 256-row tile
    const int lg = warp & 3;
    const uint32_t acc_empty_leader = leader_addr(smem_u32(&acc_empty[0]));
    int64_t j = 0;
    for (int64_t t = pair; t < n_tiles_total; t += npairs, ++j) {
      int64_t mt, nt;
      tile_coords(g, t, mt, nt);
      const int b = (int)(j & 1);
      if (!mbar_wait(smem_u32(&acc_full[b]), (uint32_t)(j >> 1) & 1u, g.err, 74)) break;
      tc_fence_after();
      const int64_t row = mt * (2 * kPHalf) + rank * kPHalf + lg * 32 + lane;
      const int64_t n0 = nt * kGN;
      const uint32_t tbase = tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(b * kGN);
#pragma unroll 1
      for (int c = 0; c < kGN; c += 32) {
        uint32_t r[32];
        tmem_ld16(tbase + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(r));
        tmem_ld16(tbase + (uint32_t)(c + 16), *reinterpret_cast<uint32_t(*)[16]>(r + 16));
        tmem_ld_wait();
        if (row < g.M) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int64_t col = n0 + c + 8 * q;
            if (col + 8 > g.N) break;
            const uint4 v = make_uint4(
                pack_bf16x2(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
            __nv_bfloat16* dst = col < g.n_split
                                     ? g.C0 + row * g.n_split + col
                                     : g.C1 + row * (g.N - g.n_split) + (col - g.n_split);
            *reinterpret_cast<uint4*>(dst) = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + (uint32_t)(b * 8));
    }
  }
  tc_fence_before();
  cluster_sync();   // no CTA leaves while its pair may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kGTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool bf16_kmajor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K,
                     uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kGK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

}  // namespace

#ifndef JMIX_GEMM_PAIR
#define JMIX_GEMM_PAIR 1
#endif

cudaError_t gemm_bf16_tn(int64_t M, int64_t N, int64_t K, const void* A, const void* B,
                         void* C0, void* C1, int64_t n_split, ErrFlags* err,
                         const ErrFlags* fold, cudaStream_t s, bool pdl) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (JMIX_GEMM_PAIR) {
    // CTA pairs: A and B tiles of 128 rows per CTA
    CUtensorMap ta, tb;
    if (!bf16_kmajor_map(&ta, A, (uint64_t)M, (uint64_t)K, kPHalf) ||
        !bf16_kmajor_map(&tb, B, (uint64_t)N, (uint64_t)K, kPHalf))
      return cudaErrorInvalidValue;
    GemmArgs g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.n_split = n_split;
    g.C0 = static_cast<__nv_bfloat16*>(C0);
    g.C1 = static_cast<__nv_bfloat16*>(C1);
    g.m_tiles = (M + 2 * kPHalf - 1) / (2 * kPHalf);
    g.n_tiles = (N + kGN - 1) / kGN;
    g.err = err;
    g.fold = fold;
    cudaError_t e = cudaFuncSetAttribute(k_gemm_bf16_pair,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = g.m_tiles * g.n_tiles;
    // as many pairs as can be resident at once (a pair needs two SMs of one GPC)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sm_count() & ~1));
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = kPSmem;
    int max_pairs = 0;
    if (cudaOccupancyMaxActiveClusters(&max_pairs, k_gemm_bf16_pair, &cfg) != cudaSuccess ||
        max_pairs <= 0)
      max_pairs = sm_count() / 2;
    const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_gemm_bf16_pair, ta, tb, g);
  }
  CUtensorMap ta, tb;
  if (!bf16_kmajor_map(&ta, A, (uint64_t)M, (uint64_t)K, kGM) ||
      !bf16_kmajor_map(&tb, B, (uint64_t)N, (uint64_t)K, kGN))
    return cudaErrorInvalidValue;
  GemmArgs g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.n_split = n_split;
  g.C0 = static_cast<__nv_bfloat16*>(C0);
  g.C1 = static_cast<__nv_bfloat16*>(C1);
  g.m_tiles = (M + kGM - 1) / kGM;
  g.n_tiles = (N + kGN - 1) / kGN;
  g.err = err;
  g.fold = fold;
  cudaError_t e = cudaFuncSetAttribute(k_gemm_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = g.m_tiles * g.n_tiles;
  const int64_t grid = tiles < sm_count() ? tiles : sm_count();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kGSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_gemm_bf16, ta, tb, g);
}

}  // namespace jmix
