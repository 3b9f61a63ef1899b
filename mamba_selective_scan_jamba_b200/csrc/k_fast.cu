// The bf16-io path of the mixer core on sm_100a.
//
// Prefill (a batch of sequences of one length, or a packed batch):
//   k_convert_weights xproj_w and dtproj_w from bf16 to fp16 (exact for |w| >=
//                     2^-14; fp16 subnormals below), unless prepared once
//                     beforehand; the conv weights as k_xproj_conv's table.
//   k_xproj_conv      u = SiLU(conv1d(x) + conv_b) in fp16, computed into the A
//                     operand of p = u . xproj_w^T on tcgen05 (TMA -> SMEM ->
//                     MMA -> TMEM); with one split over d_inner the RMSNorms in
//                     its epilogue give dt_n (fp16, the dt_proj operand) and
//                     B_n, C_n (fp32); with several each split stores its
//                     partial tile for k_norms16.
//   k_scan_fused      per (sequence, 128 channels): dt_proj on tcgen05 into
//                     TMEM, softplus, the conv + SiLU recomputed in fp32 from x,
//                     the selective scan with fp32 state in registers, the D
//                     skip, the SiLU(z) gate, the final SSM and conv states.
// Decode step (one token per row, states updated in place):
//   k_conv_step       u from x_t and each row's cached conv history; W_x to fp16.
//   k_xproj           p = u . xproj_w^T on tcgen05, split over d_inner.
//   k_norms16         sums the x_proj partials in a fixed order (so results are
//                     bitwise reproducible), then the three RMSNorms.
//   k_decode_scan     dt_proj on tcgen05 + the one-token update of the states.
// (A dt_rank that is not a multiple of 16 runs k_conv_silu16 / _packed,
// k_xproj and k_norms16 in place of k_xproj_conv.)
//
// Precision: the quantised intermediates are the two tensor-core operands, u
// for x_proj and dt_n for dt_proj, in fp16 (10 mantissa bits; their rounding
// moves y by <= ~3e-3 of max(1,|y|), against ~2e-2 for bf16 at the same
// tensor-core rate).  The scan's own u is float32, so no per-channel rounding
// decision reaches the state directly.
//
// Formulas: TransformerLens "Jamba" adapter page (mixer pipeline with the
// dt/B/C RMSNorms); aifetchly "Jamba Guide", "Inside the Mamba State-Space
// Layers" (exp(delta A) discretisation, delta B, h_t = Abar h_{t-1} + Bbar x_t,
// y_t = C_t h_t) and "Hands-On Implementation" (A = -exp(A_log),
// delta = softplus(dt_proj(.))).
#include <cuda.h>
#include <cuda_fp16.h>

#include <atomic>

#include "jmix_internal.cuh"
#include "poly_consts.cuh"
#include "sm100.cuh"

namespace jmix {
namespace {

using namespace sm100;
typedef __nv_bfloat16 bf16;

#ifndef JMIX_CONV_OCC
#define JMIX_CONV_OCC 2
#endif
// tokens per thread in k_conv_silu16: 8 for sequences (3 history rows shared by
// 8 tokens), 1 for shorter ones
constexpr int kConvG = 8;
constexpr int kXM = 128;          // x_proj tile: tokens
constexpr int kXK = 64;           // x_proj tile: channels per k-chunk (one 128-B swizzle atom)
constexpr int kXStages = 3;
#ifndef JMIX_XPROJ_CTAS  // x_proj grid target: two resident CTAs per SM
#define JMIX_XPROJ_CTAS 296
#endif
#ifndef JMIX_XSPLIT_MAX
#define JMIX_XSPLIT_MAX 16  // (32 measured ~1 us slower on a 256-row decode step)
#endif
constexpr int kMaxSplit = JMIX_XSPLIT_MAX;  // x_proj splits over d_inner, at most
#ifndef JMIX_SCAN_CHUNK
#define JMIX_SCAN_CHUNK 32
#endif
constexpr int kSQ = JMIX_SCAN_CHUNK;  // scan: tokens per chunk (the dt_proj MMA's N)
constexpr int kSC = 128;          // scan: channels per CTA
constexpr int kMaxSlabs = kMaxRank / 64;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float bf(bf16 v) { return __bfloat162float(v); }

__device__ __forceinline__ void unpack8_bf16(const uint4& q, float (&o)[8]) {
  const bf16* h = reinterpret_cast<const bf16*>(&q);
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = __bfloat162float(h[i]);
}

// Element e (0..7) of 8 packed bf16 values, as float.
__device__ __forceinline__ float bf16_lane(const uint4& v, int e) {
  const uint32_t wd = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
  return __uint_as_float((e & 1) ? (wd & 0xffff0000u) : (wd << 16));
}

__device__ __forceinline__ float clamp_half(float v) { return fminf(fmaxf(v, -65504.0f), 65504.0f); }

// Two floats to a packed fp16 pair (lo in the low 16 bits), each rounded to
// nearest even: one paired conversion instead of two single ones.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ------------------------------------------------------------------ conv + SiLU
// Thread = 8 consecutive channels x kConvG consecutive tokens of one sequence.
// All of its x rows (the 3-token history and its tokens) are loaded before any
// arithmetic, so each thread keeps ~11 16-byte loads in flight.  Threads past
// the conv range convert 8 weights each.
__device__ __forceinline__ float silu_u(float v) {
  // v * sigmoid(v); relative error ~1e-6, far below the fp16 rounding of u
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-v * kLog2e));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
  return v * r;
}

// v * sigmoid(v) with one MUFU op: 1/(1 + e) by Newton-Raphson on the FMA pipe
// from a bit-pattern initial guess (3 iterations, relative error < 2e-7 on
// [1, 8.5e37]); e is clamped so that the guess stays a normal number.
__device__ __forceinline__ float silu_newton(float v) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-v * kLog2e));
  const float den = fminf(1.0f + e, 8.5e37f);
  float r = __int_as_float(poly::RCP_MAGIC - __float_as_int(den));
  r = r * fmaf(-den, r, 2.0f);
  r = r * fmaf(-den, r, 2.0f);
  r = r * fmaf(-den, r, 2.0f);
  return v * r;
}

// The packed-batch form of k_conv_silu16: thread = 8 channels x 8 consecutive
// tokens of the packed [T, d] stream, which may span sequence boundaries.  Each
// token's sequence comes from a binary search in cu (B + 1 offsets); its taps
// before the sequence's first token come from that sequence's history (or are
// zero).  Indices are clamped so that a broken cu (reported by the scan kernel)
// cannot reach outside x or hist.  Threads past the conv range convert weights.
__global__ void __launch_bounds__(256, JMIX_CONV_OCC) k_conv_silu16_packed(
    const bf16* __restrict__ x, const bf16* __restrict__ conv_w, const bf16* __restrict__ conv_b,
    const bf16* __restrict__ hist, const int* __restrict__ cu, int64_t B, int64_t T, int64_t d,
    __half* __restrict__ u, int64_t n_conv, const bf16* __restrict__ wx, int64_t n_wx8,
    __half* __restrict__ wx16, const bf16* __restrict__ wdt, int64_t n_wdt8,
    __half* __restrict__ wdt16) {
  constexpr int G = 8, kW = kConv - 1;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid < n_conv) {
    const int64_t ncg = d >> 3;
    const int64_t cg = tid % ncg, tg = tid / ncg;
    const int64_t c0 = cg * 8, t0 = tg * G;
    const int nt = (int)((T - t0) < G ? (T - t0) : G);
    // rows[i] = packed token t0 - 3 + i (zero outside [0, T))
    uint4 rows[kW + G];
#pragma unroll
    for (int i = 0; i < kW + G; ++i) {
      const int64_t tau = t0 - kW + i;
      rows[i] = (tau >= 0 && i < kW + nt)
                    ? __ldg(reinterpret_cast<const uint4*>(x + tau * d + c0))
                    : make_uint4(0u, 0u, 0u, 0u);
    }
    // sequence of token t0: the last b with cu[b] <= t0
    int lo = 0, hi = (int)B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(cu + mid) <= t0) lo = mid; else hi = mid - 1;
    }
    const int64_t s0 = __ldg(cu + lo);
    const int64_t s_next = lo + 1 < B ? __ldg(cu + lo + 1) : T;
    // common case: every tap of the 8 tokens is inside one sequence
    const bool inner = t0 - kW >= s0 && t0 + G <= s_next;
    uint4 wq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      wq[q] = __ldg(reinterpret_cast<const uint4*>(conv_w + c0 * kConv) + q);
    const uint4 bq = __ldg(reinterpret_cast<const uint4*>(conv_b + c0));
    uint32_t outp[G][4];
    if (inner) {
      float sv_even[G];  // SiLU of the pair's even channel, per token
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float xe[kW + G];
#pragma unroll
        for (int i = 0; i < kW + G; ++i) xe[i] = bf16_lane(rows[i], e);
        float wk[kConv];
#pragma unroll
        for (int k = 0; k < kConv; ++k)
          wk[k] = bf16_lane(wq[(e * kConv + k) >> 3], (e * kConv + k) & 7);
        const float be = bf16_lane(bq, e);
#pragma unroll
        for (int i = 0; i < G; ++i) {
          float acc = be;
#pragma unroll
          for (int k = 0; k < kConv; ++k) acc = fmaf(wk[k], xe[i + k], acc);
          const float sv = clamp_half(silu_u(acc));
          if (e & 1)
            outp[i][e >> 1] = pack_half2(sv_even[i], sv);
          else
            sv_even[i] = sv;
        }
      }
    } else {
      // a sequence starts inside the window: per token, its sequence and start
#pragma unroll
      for (int i = 0; i < G; ++i) {
        int bi = lo;
        while (bi + 1 < B && __ldg(cu + bi + 1) <= t0 + i) ++bi;
        const int64_t sti = __ldg(cu + bi);
        float sv_even = 0.0f;  // SiLU of the pair's even channel
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float acc = bf16_lane(bq, e);
#pragma unroll
          for (int k = 0; k < kConv; ++k) {
            const int64_t tau = t0 + i - kW + k;
            float v = bf16_lane(rows[i + k], e);
            if (tau < sti) {
              // before the sequence's start: its history (positions -3 .. -1), else zero
              const int64_t hp = kW + (tau - sti);
              v = (hist && hp >= 0 && hp < kW) ? bf(hist[((int64_t)bi * d + c0 + e) * kW + hp])
                                               : 0.0f;
            }
            acc = fmaf(bf16_lane(wq[(e * kConv + k) >> 3], (e * kConv + k) & 7), v, acc);
          }
          const float sv = clamp_half(silu_u(acc));
          if (e & 1)
            outp[i][e >> 1] = pack_half2(sv_even, sv);
          else
            sv_even = sv;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < G; ++i) {
      if (i >= nt) break;
      *reinterpret_cast<uint4*>(u + (t0 + i) * d + c0) =
          make_uint4(outp[i][0], outp[i][1], outp[i][2], outp[i][3]);
    }
    return;
  }
  int64_t i = tid - n_conv;
  const bf16* src;
  __half* dst;
  if (i < n_wx8) {
    src = wx;
    dst = wx16;
  } else if ((i -= n_wx8) < n_wdt8) {
    src = wdt;
    dst = wdt16;
  } else {
    return;
  }
  float o[8];
  unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(src) + i), o);
  reinterpret_cast<uint4*>(dst)[i] = make_uint4(pack_half2(o[0], o[1]), pack_half2(o[2], o[3]),
                                                pack_half2(o[4], o[5]), pack_half2(o[6], o[7]));
}

template <int kConvG>
__global__ void __launch_bounds__(256, JMIX_CONV_OCC) k_conv_silu16(
    const bf16* __restrict__ x, const bf16* __restrict__ conv_w, const bf16* __restrict__ conv_b,
    const bf16* __restrict__ hist, const int* __restrict__ sidx, int64_t n_slots, int64_t B,
    int64_t L, int64_t d, __half* __restrict__ u, int64_t n_conv, const bf16* __restrict__ wx,
    int64_t n_wx8, __half* __restrict__ wx16, const bf16* __restrict__ wdt, int64_t n_wdt8,
    __half* __restrict__ wdt16) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid < n_conv) {
    const int64_t ncg = d >> 3;
    const int64_t cg = tid % ncg;
    const int64_t rest = tid / ncg;
    const int64_t nck = (L + kConvG - 1) / kConvG;
    const int64_t ck = rest % nck, b = rest / nck;
    // history row: the sequence's own, or (indexed decode step) its pool slot,
    // clamped into the pool (a bad slot is reported by the decode kernel)
    int64_t hb = b;
    if (sidx) {
      hb = __ldg(sidx + b);
      hb = hb < 0 ? 0 : (hb >= n_slots ? n_slots - 1 : hb);
    }
    const int64_t c0 = cg * 8, t0 = ck * kConvG;
    const int nt = (int)((L - t0) < kConvG ? (L - t0) : kConvG);
    constexpr int kW = kConv - 1;
    // rows[0..2] = tokens t0-3..t0-1 (history: x, the cached state or zero),
    // rows[3..] = tokens t0..t0+nt-1; kept as packed bf16 and unpacked one
    // channel at a time (fewer live registers than unpacking everything)
    uint4 rows[kW + kConvG];
#pragma unroll
    for (int i = 0; i < kW + kConvG; ++i) {
      const int64_t tau = t0 - kW + i;
      if (tau >= 0 && i < kW + nt)
        rows[i] = __ldg(reinterpret_cast<const uint4*>(x + (b * L + tau) * d + c0));
      else
        rows[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 wq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      wq[q] = __ldg(reinterpret_cast<const uint4*>(conv_w + c0 * kConv) + q);
    const uint4 bq = __ldg(reinterpret_cast<const uint4*>(conv_b + c0));
    uint32_t outp[kConvG][4];  // [token][channel pair] packed fp16x2
    float sv_even[kConvG];     // SiLU of the pair's even channel, per token
    // the 8 channels' cached conv states (3 taps each, oldest first): 48
    // contiguous bytes, 16-byte aligned since c0 is a multiple of 8
    uint4 hq[3] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                   make_uint4(0u, 0u, 0u, 0u)};
    if (t0 < kW && hist) {
      const uint4* hp = reinterpret_cast<const uint4*>(hist + (hb * d + c0) * kW);
#pragma unroll
      for (int q = 0; q < 3; ++q) hq[q] = __ldg(hp + q);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float xe[kW + kConvG];
#pragma unroll
      for (int i = 0; i < kW + kConvG; ++i) xe[i] = bf16_lane(rows[i], e);
      if (t0 < kW) {
        // taps before the sequence start: the cached conv state (zero without one);
        // history slot kW + tau of channel e is element 3 e + kW + tau of the 24
        static_assert(kConv - 1 == 3, "three history taps");
        float hv[kW];
#pragma unroll
        for (int k = 0; k < kW; ++k) hv[k] = bf16_lane(hq[(e * kW + k) >> 3], (e * kW + k) & 7);
#pragma unroll
        for (int k = 0; k < kW; ++k) {
          const int64_t slot = t0 + k;  // = kW + tau
          if (slot < kW) xe[k] = slot == 0 ? hv[0] : (slot == 1 ? hv[1] : hv[2]);
        }
      }
      float wk[kConv];
#pragma unroll
      for (int k = 0; k < kConv; ++k)
        wk[k] = bf16_lane(wq[(e * kConv + k) >> 3], (e * kConv + k) & 7);
      const float be = bf16_lane(bq, e);
#pragma unroll
      for (int i = 0; i < kConvG; ++i) {
        float acc = be;
#pragma unroll
        for (int k = 0; k < kConv; ++k) acc = fmaf(wk[k], xe[i + k], acc);
        const float sv = clamp_half(silu_u(acc));
        if (e & 1)
          outp[i][e >> 1] = pack_half2(sv_even[i], sv);
        else
          sv_even[i] = sv;
      }
    }
#pragma unroll
    for (int i = 0; i < kConvG; ++i) {
      if (i >= nt) break;
      *reinterpret_cast<uint4*>(u + (b * L + t0 + i) * d + c0) =
          make_uint4(outp[i][0], outp[i][1], outp[i][2], outp[i][3]);
    }
    return;
  }
  int64_t i = tid - n_conv;
  const bf16* src;
  __half* dst;
  if (i < n_wx8) {
    src = wx;
    dst = wx16;
  } else if ((i -= n_wx8) < n_wdt8) {
    src = wdt;
    dst = wdt16;
  } else {
    return;
  }
  float o[8];
  unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(src) + i), o);
  reinterpret_cast<uint4*>(dst)[i] = make_uint4(pack_half2(o[0], o[1]), pack_half2(o[2], o[3]),
                                                pack_half2(o[4], o[5]), pack_half2(o[6], o[7]));
}

// ------------------------------------------------------------------- x_proj
struct XprojArgs {
  int64_t T;
  int P, Ntot, N1, N2;
  int kchunks, ksplit;
  uint32_t tmem_cols;
  float* part;  // [ksplit, T, P] partial sums
  ErrFlags* err;
};

constexpr int kXThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 epilogue
constexpr int kXMaxBoxes = 9;   // the epilogue's [32 x 16] fp32 boxes per warp (N1 <= 144)

__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                                  // D format: f32
         | (0u << 7) | (0u << 10)                   // A, B format: f16
         | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Grid (2 x token tiles, d_inner splits): the R + 2N columns are cut in two
// parts of N1 (each one MMA of N <= 256, a TMEM allocation of at most 256
// columns and a 3-stage ring), so two CTAs share an SM and one's epilogue
// overlaps the other's loads.  The part is the fastest grid index: the two
// CTAs of a token tile run together and the second read of its u tile hits L2.
__global__ void __launch_bounds__(kXThreads, 2)
    k_xproj(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_w,
            const __grid_constant__ CUtensorMap tm_part, const XprojArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // (offset arithmetic on the shared array keeps its address space known, so
  // accesses through these pointers compile to shared-memory loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int a_bytes = kXM * 128;
  const int b_bytes = a.N1 * 128;
  const int col0 = (int)(blockIdx.x & 1u) * a.N1;  // this CTA's first column of p
  const int stage_bytes = a_bytes + b_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kXStages * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kXStages;
  uint64_t* acc_full = bars + 2 * kXStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kXStages + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = (int)(blockIdx.x >> 1), split = blockIdx.y;
  const int k_begin = (int)((int64_t)split * a.kchunks / a.ksplit);
  const int k_end = (int)((int64_t)(split + 1) * a.kchunks / a.ksplit);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), a.tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_u);
    prefetch_tmap(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();    // u and the fp16 W_x come from the conv kernel
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      for (int kc = k_begin, i = 0; kc < k_end; ++kc, ++i) {
        const int s = i % kXStages;
        const uint32_t ph = (uint32_t)(i / kXStages) & 1u;
        if (i >= kXStages && !mbar_wait(smem_u32(&empty[s]), ph ^ 1u, a.err, 11)) break;
        uint8_t* As = smem + s * stage_bytes;
        uint8_t* Bs = As + a_bytes;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, (uint32_t)stage_bytes);
        tma_load_2d(smem_u32(As), &tm_u, fb, kc * kXK, m_tile * kXM);
        tma_load_2d(smem_u32(Bs), &tm_w, fb, kc * kXK, col0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id1 = idesc_f16_f32(kXM, a.N1);
      for (int kc = k_begin, i = 0; kc < k_end; ++kc, ++i) {
        const int s = i % kXStages;
        const uint32_t ph = (uint32_t)(i / kXStages) & 1u;
        if (!mbar_wait(smem_u32(&full[s]), ph, a.err, 12)) break;
        tc_fence_after();
        const uint32_t ab = smem_u32(smem + s * stage_bytes);
        const uint32_t bb = ab + a_bytes;
#pragma unroll
        for (int kk = 0; kk < kXK / 16; ++kk) {
          const uint64_t ad = sw128_kmajor_desc(ab + kk * 32);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_f16(tmem, ad, sw128_kmajor_desc(bb + kk * 32), id1, acc);
        }
        umma_commit(smem_u32(&empty[s]));
      }
      umma_commit(smem_u32(acc_full));
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows, 16
    // columns at a time, into [32 rows x 16 columns] boxes of shared memory
    // (64-byte swizzle: 16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3),
    // free of bank conflicts; the stage buffers are free once the accumulator is
    // complete), which one tensor store per box writes to the split's partial
    // tile (rows past T and columns past P are not written)
    const bool ok = mbar_wait(smem_u32(acc_full), 0, a.err, 13);
    tc_fence_after();
    const int lg = warp & 3;
    const bool any = ok && k_end > k_begin;
    uint8_t* boxes = smem + lg * (kXMaxBoxes * 2048);
    const int nbox = a.N1 / 16;
    for (int j = 0; j < nbox; ++j) {
      uint32_t r[16];
      tmem_ld16(tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(j * 16), r);
      tmem_ld_wait();
      uint8_t* row = boxes + j * 2048 + lane * 64;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(row + ((q ^ ((lane >> 1) & 3)) << 4)) =
            any ? make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3])
                : make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();  // the boxes, before the tensor stores read them
    __syncwarp();
    if (lane == 0) {
      for (int j = 0; j < nbox; ++j)
        tma_store_3d(&tm_part, smem_u32(boxes + j * 2048), col0 + j * 16,
                     m_tile * kXM + lg * 32, split);
      bulk_commit();
      bulk_wait_all();  // the partial tile written (and the boxes read) before the CTA ends
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

// -------------------------------------------------------------------- norms
// TPB tokens per block: p[j] = sum of the ksplit partial rows in ascending
// split order (threads over (token, column) pairs), then per token the norms
// (one warp: dt over R; B and C over N).  dt_n is written in fp16, the dt_proj
// operand type.  TPB = 8 for many tokens, 1 when few tokens carry many splits.
constexpr int kMaxP = kMaxRank + 2 * kN;
constexpr int kNormThreads = 256;

template <typename W, int TPB>
__global__ void __launch_bounds__(kNormThreads) k_norms16(
    const float* __restrict__ part, int ksplit, const W* __restrict__ wdt,
    const W* __restrict__ wb, const W* __restrict__ wc, int64_t Tn, int R, float eps,
    __half* __restrict__ dtn, float* __restrict__ bc) {
  __shared__ float rows[TPB][kMaxP];
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  // the norm weights this lane applies (inputs: loaded before the wait)
  float wk[kMaxRank / 32];
#pragma unroll
  for (int j = 0; j < kMaxRank / 32; ++j) {
    const int k = lane + 32 * j;
    wk[j] = k < R ? (float)__ldg(wdt + k) : 0.0f;
  }
  const float wv = lane < kN ? (float)__ldg(wb + lane) : (float)__ldg(wc + lane - kN);
  grid_dep_wait();    // the partial sums come from x_proj
  grid_dep_launch();
  const int64_t g0 = (int64_t)blockIdx.x * TPB;
  const int P = R + 2 * kN;
  const int64_t stride = Tn * P;
  for (int idx = threadIdx.x; idx < TPB * P; idx += kNormThreads) {
    const int tl = idx / P, j = idx - tl * P;
    const int64_t g = g0 + tl;
    if (g >= Tn) continue;
    const float* src = part + g * P + j;
    // every split's value is loaded before the sum (one memory round trip);
    // the sum still runs in ascending split order
    float v[kMaxSplit];
#pragma unroll
    for (int sp = 0; sp < kMaxSplit; ++sp) v[sp] = sp < ksplit ? src[sp * stride] : 0.0f;
    float acc = v[0];
#pragma unroll
    for (int sp = 1; sp < kMaxSplit; ++sp)
      if (sp < ksplit) acc += v[sp];
    rows[tl][j] = acc;
  }
  __syncthreads();
  for (int tl = wi; tl < TPB; tl += kNormThreads / 32) {
    const int64_t g = g0 + tl;
    if (g >= Tn) break;
    const float* row = rows[tl];
    float ss = 0.f;
    for (int k = lane; k < R; k += 32) ss = fmaf(row[k], row[k], ss);
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)R + eps);
#pragma unroll
    for (int j = 0; j < kMaxRank / 32; ++j) {
      const int k = lane + 32 * j;
      if (k < R) dtn[g * R + k] = __float2half_rn(row[k] * inv * wk[j]);
    }
    const float v = row[R + lane];
    float s2 = v * v;
#pragma unroll
    for (int o = 8; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    const float inv2 = 1.0f / sqrtf(s2 / (float)kN + eps);
    bc[g * 2 * kN + lane] = v * inv2 * wv;
  }
}

// One warp per token, for at most 4 splits: every load of the row (9 columns x
// up to 4 splits per lane) is issued before the sums, which then run in
// ascending split order; then the norms as in k_norms16.
template <typename W>
__global__ void __launch_bounds__(256) k_norms16_warp(
    const float* __restrict__ part, int ksplit, const W* __restrict__ wdt,
    const W* __restrict__ wb, const W* __restrict__ wc, int64_t Tn, int R, float eps,
    __half* __restrict__ dtn, float* __restrict__ bc) {
  constexpr int kCols = kMaxP / 32;
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  // the norm weights this lane applies (inputs: loaded before the wait)
  float wk[kCols];
#pragma unroll
  for (int jj = 0; jj < kCols; ++jj) {
    const int j = lane + 32 * jj;
    wk[jj] = j < R ? (float)__ldg(wdt + j) : 0.0f;
  }
  const float wv = lane < kN ? (float)__ldg(wb + lane) : (float)__ldg(wc + lane - kN);
  grid_dep_wait();    // the partial sums come from x_proj
  grid_dep_launch();
  const int64_t g = (int64_t)blockIdx.x * 8 + wi;
  if (g >= Tn) return;
  const int P = R + 2 * kN;
  const int64_t stride = Tn * P;
  float v[kCols][4];
#pragma unroll
  for (int jj = 0; jj < kCols; ++jj) {
    const int j = lane + 32 * jj;
#pragma unroll
    for (int sp = 0; sp < 4; ++sp)
      v[jj][sp] = (j < P && sp < ksplit) ? part[sp * stride + g * P + j] : 0.0f;
  }
  float row[kCols];
#pragma unroll
  for (int jj = 0; jj < kCols; ++jj) {
    float acc = v[jj][0];
#pragma unroll
    for (int sp = 1; sp < 4; ++sp)
      if (sp < ksplit) acc += v[jj][sp];
    row[jj] = acc;
  }
  // dt occupies columns [0, R): lanes hold row[jj] for j = lane + 32 jj
  float ss = 0.f;
#pragma unroll
  for (int jj = 0; jj < kCols; ++jj)
    if (lane + 32 * jj < R) ss = fmaf(row[jj], row[jj], ss);
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)R + eps);
#pragma unroll
  for (int jj = 0; jj < kCols; ++jj) {
    const int j = lane + 32 * jj;
    if (j < R) dtn[g * R + j] = __float2half_rn(row[jj] * inv * wk[jj]);
  }
  // B and C occupy columns [R, R + 32): R is a multiple of 8, so pick them up by shuffles
  float bcv = 0.f;
#pragma unroll
  for (int jj = 0; jj < kCols; ++jj) {
    // column R + lane lives in lane (R + lane) % 32 of slot (R + lane) / 32
    const int src_j = R + lane;
    const float t = __shfl_sync(0xffffffffu, row[jj], src_j & 31);
    if ((src_j >> 5) == jj) bcv = t;
  }
  float s2 = bcv * bcv;
#pragma unroll
  for (int o = 8; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  const float inv2 = 1.0f / sqrtf(s2 / (float)kN + eps);
  bc[g * 2 * kN + lane] = bcv * inv2 * wv;
}

// ------------------------------------------------ conv + SiLU inside x_proj
// The prefill form of steps 1-3 (sequences of one length, T = B L tokens, or a
// packed batch whose tokens find their sequence in cu):
// x_proj's A operand u = SiLU(conv(x)) is computed in shared memory from TMA
// tiles of x, so u never goes through global memory (the scan recomputes its
// own u in float32).  Grid (token tiles of 128, splits of d_inner); each CTA
// computes all R + 2N columns of its tiles as two MMAs of N1 columns.
//   warp 0      TMA: per 64-channel chunk the x rows m0 - 3 .. m0 + 127 (one
//               box of 131 rows; rows before token 0 and past T read as zero),
//               the chunk's conv weights and biases (bulk copies) and its two
//               W_x boxes;
//   warp 1      TMEM owner and MMA issuer (2 x 4 tcgen05.mma per chunk);
//   warps 2-    conv (JMIX_XCONV_WARPS of them; with JMIX_XCONV_GROUPS > 1 in
//               groups that take alternate chunks): thread = 8 channels x kFG
//               tokens (4 with 8 warps in one group), each token's u stored as
//               soon as it is computed.
//               The kFG + 3 x rows come from the stage, taps before a
//               sequence's first token from its history (or zero); u in fp16
//               goes into the 128-byte-swizzled A stage, rounded exactly as
//               k_conv_silu16 rounds it.  Then the epilogue.
// With one split the epilogue applies the RMSNorms itself (thread = token row
// of TMEM, the sums of squares taken in the order of k_norms16_warp's
// reductions) and writes dt_n and B, C; with several it writes the fp32
// partial sums that k_norms16 adds up.
#ifndef JMIX_XCONV_WARPS
#define JMIX_XCONV_WARPS 8  // conv warps (8: 4 tokens per thread, 16: 2)
#endif
#ifndef JMIX_XCONV_GROUPS
#define JMIX_XCONV_GROUPS 1  // conv warp groups taking alternate chunks (2 measured slower)
#endif
constexpr int kFConvWarps = JMIX_XCONV_WARPS;
constexpr int kFGroups = JMIX_XCONV_GROUPS;
constexpr int kFGroupWarps = kFConvWarps / kFGroups;
constexpr int kFG = kXM * (kXK / 8) / (kFGroupWarps * 32);  // tokens per conv thread
constexpr int kFThreads = 64 + 32 * kFConvWarps;
constexpr int kFStages = 3;
constexpr int kFXRows = kXM + kConv - 1;                    // 131 x rows per chunk
constexpr int kFXBytes = kFXRows * kXK * 2;                 // 16768 B
// the chunk's conv weights and biases in float32, laid out for the conv threads
// (see k_conv_table): 8 weight units and 2 bias units of 16 B per 8 channels
constexpr int kFTabUnits = (kXK / 8) * 10;                  // 80
constexpr int kFTabBytes = kFTabUnits * 16;                 // 1280 B
constexpr int kFXStride = (kFXBytes + kFTabBytes + 1023) / 1024 * 1024;  // 18 KB
constexpr int kFABytes = kXM * kXK * 2;                     // 16 KB u tile
constexpr int kFMaxN1 = (kMaxRank + 2 * kN) / 2;            // 144
constexpr int kFBMax = 2 * kFMaxN1 * kXK * 2;               // 36 KB of W_x rows
constexpr int kFSmem = 1024 + kFStages * (kFABytes + kFBMax + kFXStride) + 256;
static_assert(kFSmem <= 227 * 1024, "fused x_proj stage ring exceeds shared memory");
static_assert(8 * kXMaxBoxes * 2048 <= kFStages * (kFABytes + kFBMax),
              "the epilogue's partial-sum boxes exceed the A and B stages");
static_assert(kFGroupWarps * kFGroups == kFConvWarps &&
                  kFGroupWarps * 32 * kFG == kXM * (kXK / 8),
              "a group's conv threads = kFG-token x 8-channel cells of a chunk");

// The weight preparation of a prefill: W_x and W_dt to fp16 (unless prepared
// once beforehand), 8 weights per thread, and the conv weights and biases as
// k_xproj_conv's float32 table: per 64-channel chunk kFTabUnits 16-byte units,
// unit u * 8 + g (u < 8) = the taps 2 (u % 2), 2 (u % 2) + 1 of the channel pair
// 2 (u / 2), 2 (u / 2) + 1 of the chunk's channel group g (8 channels), as
// (w[c][k], w[c + 1][k], w[c][k + 1], w[c + 1][k + 1]); unit 64 + v * 8 + g =
// the biases of channels 4 v .. 4 v + 3 of group g.  Zeros past d.
__global__ void __launch_bounds__(256) k_convert_weights(
    const bf16* __restrict__ wx, int64_t n_wx8, __half* __restrict__ wx16,
    const bf16* __restrict__ wdt, int64_t n_wdt8, __half* __restrict__ wdt16,
    const bf16* __restrict__ conv_w, const bf16* __restrict__ conv_b, int64_t d,
    float4* __restrict__ ctab, int64_t n_tab, unsigned* __restrict__ zero_w, int n_zero_w) {
  // the kernels before this one may still read the workspace; the call's error
  // header and scheduler words are cleared here (the later kernels of the call
  // start after this one has completed)
  grid_dep_wait();
  if (blockIdx.x == 0)
    for (int z = threadIdx.x; z < n_zero_w; z += blockDim.x) zero_w[z] = 0u;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bf16* src = nullptr;
  __half* dst = nullptr;
  if (i < n_wx8) {
    src = wx;
    dst = wx16;
  } else if ((i -= n_wx8) < n_wdt8) {
    src = wdt;
    dst = wdt16;
  } else if ((i -= n_wdt8) < n_tab) {
    const int64_t kc = i / kFTabUnits;
    const int r = (int)(i - kc * kFTabUnits);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < 64) {
      const int u = r >> 3, g = r & 7, k = 2 * (u & 1);
      const int64_t c = kc * kXK + g * 8 + 2 * (u >> 1);
      if (c < d)  // d is a multiple of 8: both channels of the pair exist, or neither
        v = make_float4(bf(conv_w[c * kConv + k]), bf(conv_w[(c + 1) * kConv + k]),
                        bf(conv_w[c * kConv + k + 1]), bf(conv_w[(c + 1) * kConv + k + 1]));
    } else {
      const int hv = (r - 64) >> 3, g = (r - 64) & 7;
      const int64_t c = kc * kXK + g * 8 + 4 * hv;
      if (c < d)
        v = make_float4(bf(conv_b[c]), bf(conv_b[c + 1]), bf(conv_b[c + 2]), bf(conv_b[c + 3]));
    }
    ctab[i] = v;
    return;
  } else {
    return;
  }
  float o[8];
  unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(src) + i), o);
  reinterpret_cast<uint4*>(dst)[i] = make_uint4(pack_half2(o[0], o[1]), pack_half2(o[2], o[3]),
                                                pack_half2(o[4], o[5]), pack_half2(o[6], o[7]));
}

struct XconvArgs {
  int64_t T, L, d;
  int P, N1, R;
  int kchunks, ksplit;
  uint32_t tmem_cols;
  const float4* ctab;  // [kchunks * kFTabUnits] the conv weights and biases (k_conv_table)
  const bf16* hist;    // [B, d, 3] conv history of each sequence, or null (zeros)
  const int* cu;       // packed batch: [B + 1] token offsets of the sequences, or null
  int64_t nseq;        // packed batch: sequences B
  float* part;         // [ksplit, T, P] partial sums (ksplit > 1)
  const bf16* dtn_w;   // [R]
  const bf16* bn_w;    // [N]
  const bf16* cn_w;    // [N]
  float eps;
  __half* dtn;         // [T, R] (ksplit == 1)
  float* bc;           // [T, 2N] (ksplit == 1)
  ErrFlags* err;
};

// Channels (2q, 2q + 1) of 8 packed bf16 values as a float pair.
__device__ __forceinline__ float2 bf16_pair(const uint4& v, int q) {
  const uint32_t w = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

#ifndef JMIX_XCONV_SILU1
#define JMIX_XCONV_SILU1 0  // 1: the reciprocal by Newton steps on the FMA pipe (one MUFU op)
#endif
// SiLU of a pair, clamped to the fp16 range and packed as fp16x2: the same
// operations, in the same order, as clamp_half(silu_u(v)) on each element
// (with JMIX_XCONV_SILU1, as silu_newton), one saturating conversion for the
// clamp and the rounding.
__device__ __forceinline__ uint32_t silu_u_half2(float2 v) {
  const float2 t = __fmul2_rn(v, make_float2(-kLog2e, -kLog2e));
  float2 e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.x) : "f"(t.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.y) : "f"(t.y));
  float2 den = __fadd2_rn(make_float2(1.0f, 1.0f), e);
#if JMIX_XCONV_SILU1
  den = make_float2(fminf(den.x, 8.5e37f), fminf(den.y, 8.5e37f));
  r = make_float2(__int_as_float(poly::RCP_MAGIC - __float_as_int(den.x)),
                  __int_as_float(poly::RCP_MAGIC - __float_as_int(den.y)));
  const float2 nd = make_float2(-den.x, -den.y), two = make_float2(2.0f, 2.0f);
  r = __fmul2_rn(r, __ffma2_rn(nd, r, two));
  r = __fmul2_rn(r, __ffma2_rn(nd, r, two));
  r = __fmul2_rn(r, __ffma2_rn(nd, r, two));
#else
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(den.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(den.y));
#endif
  const float2 s = __fmul2_rn(v, r);
  // round to fp16, saturating to +-65504: the same bits as clamp_half then
  // rounding for every number (a NaN stays NaN here)
  uint32_t h;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(s.y), "f"(s.x));
  return h;
}

// ------------------------------------------------- conv + SiLU of a decode step
// One token per row (L = 1): every tap but the last comes from the row's cached
// history (its pool slot for an indexed step, clamped into the pool; a bad slot
// is reported and skipped by the decode kernel).  Thread = 8 channels of
// kStepRows rows, so the channels' conv weights are unpacked once for all of
// them; all of its loads are issued before any arithmetic, and the index
// arithmetic is 32-bit (the host checks the sizes).  u is rounded to fp16 with
// the same operations, in the same order, as k_conv_silu16 (pairs of channels).
// Threads past the conv range convert 8 W_x weights each to fp16.
#ifndef JMIX_STEP_ROWS
#define JMIX_STEP_ROWS 4
#endif
#ifndef JMIX_STEP_CVT
#define JMIX_STEP_CVT 4  // 16-byte groups of W_x converted per thread
#endif
#ifndef JMIX_STEP_OCC
#define JMIX_STEP_OCC 2
#endif
constexpr int kStepRows = JMIX_STEP_ROWS;
constexpr int kStepCvt = JMIX_STEP_CVT;

__global__ void __launch_bounds__(256, JMIX_STEP_OCC) k_conv_step(
    const bf16* __restrict__ x, const bf16* __restrict__ conv_w, const bf16* __restrict__ conv_b,
    const bf16* __restrict__ hist, const int* __restrict__ sidx, int n_slots, int B, int d,
    __half* __restrict__ u, int n_conv, const bf16* __restrict__ wx, int n_wx8,
    __half* __restrict__ wx16, unsigned* __restrict__ zero_w, int n_zero_w) {
  // x_t and the conv states may come from the kernels before this one; the
  // step's error header is cleared here (the later kernels of the step start
  // after this one has completed)
  grid_dep_wait();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero_w; i += blockDim.x) zero_w[i] = 0u;
  const int tid = (int)(blockIdx.x * blockDim.x + threadIdx.x);
  if (tid < n_conv) {
    constexpr int kW = kConv - 1;
    const int ncg = d >> 3;
    const int rg = tid / ncg, cg = tid - rg * ncg;
    const int c0 = cg * 8, b0 = rg * kStepRows;
    uint4 xq[kStepRows], hq[kStepRows][kW];
#pragma unroll
    for (int r = 0; r < kStepRows; ++r) {
      const int b = b0 + r;
      xq[r] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int q = 0; q < kW; ++q) hq[r][q] = make_uint4(0u, 0u, 0u, 0u);
      if (b < B) {
        xq[r] = __ldg(reinterpret_cast<const uint4*>(x + (int64_t)b * d + c0));
        if (hist) {
          int hb = b;
          if (sidx) {
            hb = __ldg(sidx + b);
            hb = hb < 0 ? 0 : (hb >= n_slots ? n_slots - 1 : hb);
          }
          // the 8 channels' 3 taps each, oldest first: 48 contiguous bytes
          const uint4* hp = reinterpret_cast<const uint4*>(hist + ((int64_t)hb * d + c0) * kW);
#pragma unroll
          for (int q = 0; q < kW; ++q) hq[r][q] = __ldg(hp + q);
        }
      }
    }
    uint4 wq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) wq[q] = __ldg(reinterpret_cast<const uint4*>(conv_w + c0 * kConv) + q);
    const uint4 bq = __ldg(reinterpret_cast<const uint4*>(conv_b + c0));
    float2 w2[4][kConv], b2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int k = 0; k < kConv; ++k) {
        const int e0 = (2 * q) * kConv + k, e1 = (2 * q + 1) * kConv + k;
        w2[q][k] = make_float2(bf16_lane(wq[e0 >> 3], e0 & 7), bf16_lane(wq[e1 >> 3], e1 & 7));
      }
      b2[q] = make_float2(bf16_lane(bq, 2 * q), bf16_lane(bq, 2 * q + 1));
    }
#pragma unroll
    for (int r = 0; r < kStepRows; ++r) {
      uint32_t out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 acc = b2[q];
#pragma unroll
        for (int k = 0; k < kW; ++k) {
          const int e0 = (2 * q) * kW + k, e1 = (2 * q + 1) * kW + k;
          acc = __ffma2_rn(w2[q][k],
                           make_float2(bf16_lane(hq[r][e0 >> 3], e0 & 7),
                                       bf16_lane(hq[r][e1 >> 3], e1 & 7)),
                           acc);
        }
        acc = __ffma2_rn(w2[q][kW], bf16_pair(xq[r], q), acc);
        out[q] = silu_u_half2(acc);
      }
      const int b = b0 + r;
      if (b < B)
        *reinterpret_cast<uint4*>(u + (int64_t)b * d + c0) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    return;
  }
  // kStepCvt groups of 8 weights per thread, every load before the stores
  const int i0 = (tid - n_conv) * kStepCvt;
  uint4 wv[kStepCvt];
#pragma unroll
  for (int j = 0; j < kStepCvt; ++j)
    if (i0 + j < n_wx8) wv[j] = __ldg(reinterpret_cast<const uint4*>(wx) + i0 + j);
#pragma unroll
  for (int j = 0; j < kStepCvt; ++j) {
    if (i0 + j >= n_wx8) break;
    float o[8];
    unpack8_bf16(wv[j], o);
    reinterpret_cast<uint4*>(wx16)[i0 + j] =
        make_uint4(pack_half2(o[0], o[1]), pack_half2(o[2], o[3]), pack_half2(o[4], o[5]),
                   pack_half2(o[6], o[7]));
  }
}

__global__ void __launch_bounds__(kFThreads, 1)
    k_xproj_conv(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_part, const XconvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* As = smem;                          // [stages] u tiles (128-byte swizzle)
  uint8_t* Bs = As + kFStages * kFABytes;      // [stages] W_x boxes (128-byte swizzle)
  uint8_t* Xs = Bs + kFStages * kFBMax;        // [stages] x rows (plain)
  uint64_t* bars = reinterpret_cast<uint64_t*>(Xs + kFStages * kFXStride);
  uint64_t* full = bars;                       // [stages] x rows and W_x landed
  uint64_t* afull = bars + kFStages;           // [stages] u tile written (conv warps)
  uint64_t* mdone = bars + 2 * kFStages;       // [stages] the MMAs have read the stage
  uint64_t* acc_full = bars + 3 * kFStages;    // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kXM;
  const int split = blockIdx.y;
  const int k_begin = (int)((int64_t)split * a.kchunks / a.ksplit);
  const int k_end = (int)((int64_t)(split + 1) * a.kchunks / a.ksplit);
  const uint32_t half_b = (uint32_t)(a.N1 * kXK * 2);  // bytes of one W_x box

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&afull[s]), kFGroupWarps);
      mbar_init(smem_u32(&mdone[s]), 1);
    }
    mbar_init(smem_u32(acc_full), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), a.tmem_cols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();    // the fp16 W_x may come from the kernel before this one
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      for (int kc = k_begin, i = 0; kc < k_end; ++kc, ++i) {
        const int s = i % kFStages;
        if (i >= kFStages &&
            !mbar_wait(smem_u32(&mdone[s]), (uint32_t)((i / kFStages) - 1) & 1u, a.err, 85))
          break;
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, (uint32_t)(kFXBytes + kFTabBytes) + 2 * half_b);
        uint8_t* xst = Xs + s * kFXStride;
        tma_load_2d(smem_u32(xst), &tm_x, fb, kc * kXK, (int32_t)(m0 - (kConv - 1)));
        // the chunk's conv weights and biases (zeros for channels past d)
        bulk_load(smem_u32(xst + kFXBytes), a.ctab + (int64_t)kc * kFTabUnits, kFTabBytes, fb);
        const uint32_t bs = smem_u32(Bs + s * kFBMax);
        tma_load_2d(bs, &tm_w, fb, kc * kXK, 0);
        tma_load_2d(bs + half_b, &tm_w, fb, kc * kXK, a.N1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_f16_f32(kXM, a.N1);
      for (int kc = k_begin, i = 0; kc < k_end; ++kc, ++i) {
        const int s = i % kFStages;
        const uint32_t ph = (uint32_t)(i / kFStages) & 1u;
        if (!mbar_wait(smem_u32(&afull[s]), ph, a.err, 86)) break;
        if (!mbar_wait(smem_u32(&full[s]), ph, a.err, 87)) break;
        tc_fence_after();
        const uint32_t ab = smem_u32(As + s * kFABytes), bb = smem_u32(Bs + s * kFBMax);
#pragma unroll
        for (int kk = 0; kk < kXK / 16; ++kk) {
          const uint64_t ad = sw128_kmajor_desc(ab + kk * 32);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_f16(tmem, ad, sw128_kmajor_desc(bb + kk * 32), id, acc);
          umma_f16(tmem + (uint32_t)a.N1, ad, sw128_kmajor_desc(bb + half_b + kk * 32), id, acc);
        }
        umma_commit(smem_u32(&mdone[s]));
      }
      umma_commit(smem_u32(acc_full));
    }
  } else {
    // ---- conv: group grp takes chunks grp, grp + kFGroups, ...; thread =
    // channels cg*8 .. +7 of the chunk, tile rows kFG tg .. + kFG - 1
    const int grp = (warp - 2) / kFGroupWarps;
    const int ct = threadIdx.x - 64 - grp * kFGroupWarps * 32;
    const int cg = ct & 7, tg = ct >> 3;
    constexpr int kW = kConv - 1;
    // sequence and position of the thread's kFG tokens (the same for every
    // chunk); a token at position < 3 takes taps from its sequence's history
    int tseq[kFG];  // (a sequence index)
    int tpos[kFG];
    bool tedge[kFG], edge = false;
#pragma unroll
    for (int ti = 0; ti < kFG; ++ti) {
      const int64_t g = m0 + kFG * tg + ti;
      if (a.cu) {
        // packed batch: the last sequence whose first token is at or before g
        // (clamped to [0, B); a broken cu is reported by the scan kernel)
        int lo = 0, hi = (int)a.nseq - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (__ldg(a.cu + mid) <= g) lo = mid; else hi = mid - 1;
        }
        tseq[ti] = lo;
        tpos[ti] = (int)(g - __ldg(a.cu + lo));
      } else {
        tseq[ti] = (int)(g / a.L);
        tpos[ti] = (int)(g - (int64_t)tseq[ti] * a.L);
      }
      tedge[ti] = g < a.T && tpos[ti] >= 0 && tpos[ti] < kW;
      edge |= tedge[ti];
    }
    // When the thread's first token is at position < 3 and all its tokens lie
    // in that sequence (every sequence start when kFG divides L), the x rows
    // before the sequence are needed by this thread alone: they are replaced by
    // the history rows once per chunk, and the common path computes the rest.
    // Other layouts of sequence starts recompute their edge tokens (slow).
    const bool sub = tedge[0] && tseq[kFG - 1] == tseq[0];
    const bool slow = edge && !sub;
    for (int kc = k_begin + grp, i = grp; kc < k_end; kc += kFGroups, i += kFGroups) {
      const int s = i % kFStages;
      const uint32_t ph = (uint32_t)(i / kFStages) & 1u;
      const int64_t c0 = (int64_t)kc * kXK + cg * 8;
      const bool cin = c0 < a.d;  // d is a multiple of 8: all 8 channels exist, or none
      if (!mbar_wait(smem_u32(&full[s]), ph, a.err, 88)) break;
      // this thread's 8 channels' conv weights and biases in float32, as pairs
      // of channels: unit u * 8 + cg of the stage's table, so that the 8 threads
      // of a quarter warp read 128 consecutive bytes
      const uint8_t* xst = Xs + s * kFXStride;
      const float4* tab = reinterpret_cast<const float4*>(xst + kFXBytes);
      float2 w2[4][kConv], b2[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int kh = 0; kh < kConv / 2; ++kh) {
          const float4 v = tab[(q * 2 + kh) * 8 + cg];
          w2[q][2 * kh] = make_float2(v.x, v.y);
          w2[q][2 * kh + 1] = make_float2(v.z, v.w);
        }
      }
#pragma unroll
      for (int hv = 0; hv < 2; ++hv) {
        const float4 v = tab[64 + hv * 8 + cg];
        b2[2 * hv] = make_float2(v.x, v.y);
        b2[2 * hv + 1] = make_float2(v.z, v.w);
      }
      const uint8_t* xs = xst + (kFG * tg) * (kXK * 2) + cg * 16;
      uint4 xr[kFG + kW];
#pragma unroll
      for (int j = 0; j < kFG + kW; ++j) xr[j] = *reinterpret_cast<const uint4*>(xs + j * (kXK * 2));
      // token ti's u into the A stage: row r, 16-byte chunk cg at cg ^ (r % 8)
      // (128-byte swizzle); zeros for channels past d
      uint8_t* at = As + s * kFABytes;
      auto store_u = [&](int ti, const uint32_t (&o)[4]) {
        const int r = kFG * tg + ti;
        *reinterpret_cast<uint4*>(at + r * (kXK * 2) + ((cg ^ (r & 7)) << 4)) =
            cin ? make_uint4(o[0], o[1], o[2], o[3]) : make_uint4(0u, 0u, 0u, 0u);
      };
      if (sub) {
        // raw row j < 3 - tpos[0] holds position tpos[0] - 3 + j < 0 of the
        // sequence: history slot tpos[0] + j (channel e's slots sit at 3 e ..)
        uint4 hq[3] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u),
                       make_uint4(0u, 0u, 0u, 0u)};
        if (cin && a.hist) {
          const uint4* hp =
              reinterpret_cast<const uint4*>(a.hist + ((int64_t)tseq[0] * a.d + c0) * kW);
#pragma unroll
          for (int q = 0; q < 3; ++q) hq[q] = __ldg(hp + q);
        }
        const uint32_t* hw = reinterpret_cast<const uint32_t*>(hq);
        uint4 hrows[kW];  // [slot]: the 8 channels' values at that history slot
#pragma unroll
        for (int sl = 0; sl < kW; ++sl) {
          uint32_t wv[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int i0 = 3 * (2 * w) + sl, i1 = 3 * (2 * w + 1) + sl;  // 16-bit elements
            const uint32_t lo = (hw[i0 >> 1] >> (16 * (i0 & 1))) & 0xffffu;
            const uint32_t hi = (hw[i1 >> 1] >> (16 * (i1 & 1))) & 0xffffu;
            wv[w] = lo | (hi << 16);
          }
          hrows[sl] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
#pragma unroll
        for (int j = 0; j < kW; ++j) {
          if (j < kW - tpos[0]) {
            const int sl = tpos[0] + j;
            xr[j] = sl == 0 ? hrows[0] : (sl == 1 ? hrows[1] : hrows[2]);
          }
        }
      }
      // every token from the kFG + 3 x rows (one basic block: the chains interleave)
#pragma unroll
      for (int ti = 0; ti < kFG; ++ti) {
        uint32_t o[4];  // channel pairs as fp16x2
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 acc = b2[q];
#pragma unroll
          for (int k = 0; k < kConv; ++k) acc = __ffma2_rn(w2[q][k], bf16_pair(xr[ti + k], q), acc);
          o[q] = silu_u_half2(acc);
        }
        store_u(ti, o);
      }
      if (slow) {
        // rare: tokens at positions 0-2 of their sequence in a thread that
        // also holds tokens of the sequence before, again with the taps before
        // the sequence's first token from its history (or zero)
#pragma unroll
        for (int ti = 0; ti < kFG; ++ti) {
          if (!tedge[ti]) continue;
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float2 acc = b2[q];
#pragma unroll
            for (int k = 0; k < kConv; ++k) {
              float2 xv = bf16_pair(xr[ti + k], q);
              if (k < kW && tpos[ti] + k < kW) {
                xv = make_float2(0.f, 0.f);
                if (a.hist) {
                  const bf16* hp =
                      a.hist + ((int64_t)tseq[ti] * a.d + c0 + 2 * q) * kW + tpos[ti] + k;
                  xv = make_float2(bf(hp[0]), bf(hp[kW]));
                }
              }
              acc = __ffma2_rn(w2[q][k], xv, acc);
            }
            o[q] = silu_u_half2(acc);
          }
          store_u(ti, o);  // (over the first pass's value)
        }
      }
      fence_proxy_async_smem();  // u in the stage, before the tensor cores read it
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&afull[s]));
    }

    // ---- epilogue (warps 2-9): warp w reads TMEM lanes 32 (w % 4) .. + 31 = tile rows
    if (warp < 10) {
      const bool ok = mbar_wait(smem_u32(acc_full), 0, a.err, 89);
      tc_fence_after();
      const int lg = warp & 3;
      const bool lower = warp < 6;  // warps 2-5, else 6-9: two warps per lane group
      const int64_t g = m0 + lg * 32 + lane;  // this thread's token
      const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
      if (a.ksplit == 1) {
        if (lower) {
          // dt: sum of squares as k_norms16_warp takes it (lane l: columns l + 32 j
          // in order, then the xor-butterfly over the lanes)
          float ps[32];
#pragma unroll
          for (int l = 0; l < 32; ++l) ps[l] = 0.0f;
#pragma unroll 1
          for (int c = 0; c < a.R; c += 32) {
            uint32_t r0[16], r1[16];
            const bool two = c + 16 < a.R;  // R is a multiple of 16
            tmem_ld16(trow + (uint32_t)c, r0);
            if (two) tmem_ld16(trow + (uint32_t)(c + 16), r1);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float v = __uint_as_float(r0[e]);
              ps[e] = fmaf(v, v, ps[e]);
            }
            if (two) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float v = __uint_as_float(r1[e]);
                ps[16 + e] = fmaf(v, v, ps[16 + e]);
              }
            }
          }
#pragma unroll
          for (int o = 16; o; o >>= 1)
#pragma unroll
            for (int l = 0; l < o; ++l) ps[l] = ps[l] + ps[l + o];
          const float inv = 1.0f / sqrtf(ps[0] / (float)a.R + a.eps);
#pragma unroll 1
          for (int c = 0; c < a.R; c += 16) {
            uint32_t r[16];
            tmem_ld16(trow + (uint32_t)c, r);
            tmem_ld_wait();
            if (ok && g < a.T) {
              uint32_t hw[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                hw[e] = pack_half2(__uint_as_float(r[2 * e]) * inv * bf(a.dtn_w[c + 2 * e]),
                                   __uint_as_float(r[2 * e + 1]) * inv * bf(a.dtn_w[c + 2 * e + 1]));
              uint4* dst = reinterpret_cast<uint4*>(a.dtn + g * a.R + c);
              dst[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              dst[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            }
          }
        } else {
          // B (columns R .. R + 15) and C (R + 16 .. R + 31): 16-lane butterflies
          uint32_t rv[2][16];
          tmem_ld16(trow + (uint32_t)a.R, rv[0]);
          tmem_ld16(trow + (uint32_t)(a.R + 16), rv[1]);
          tmem_ld_wait();
          if (ok && g < a.T) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float sq[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float v = __uint_as_float(rv[h][e]);
                sq[e] = v * v;
              }
#pragma unroll
              for (int o = 8; o; o >>= 1)
#pragma unroll
                for (int l = 0; l < o; ++l) sq[l] = sq[l] + sq[l + o];
              const float inv2 = 1.0f / sqrtf(sq[0] / (float)kN + a.eps);
              const bf16* wn = h ? a.cn_w : a.bn_w;
              float4* dst = reinterpret_cast<float4*>(a.bc + g * 2 * kN + h * kN);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_float4(__uint_as_float(rv[h][4 * e]) * inv2 * bf(wn[4 * e]),
                                     __uint_as_float(rv[h][4 * e + 1]) * inv2 * bf(wn[4 * e + 1]),
                                     __uint_as_float(rv[h][4 * e + 2]) * inv2 * bf(wn[4 * e + 2]),
                                     __uint_as_float(rv[h][4 * e + 3]) * inv2 * bf(wn[4 * e + 3]));
            }
          }
        }
      } else {
        // partial sums: columns [0, N1) by warps 2-5, [N1, 2 N1) by warps 6-9,
        // 16 at a time into [32 rows x 16 columns] boxes of shared memory
        // (64-byte swizzle: 16-byte chunk q of row r at chunk q ^ ((r >> 1) & 3);
        // the A and B stages are free once the accumulator is complete), which
        // one tensor store per box writes (rows past T, columns past P are not)
        const int cbeg = lower ? 0 : a.N1;
        uint8_t* boxes = smem + (warp - 2) * (kXMaxBoxes * 2048);
        const int nbox = a.N1 / 16;
        for (int j = 0; j < nbox; ++j) {
          uint32_t r[16];
          tmem_ld16(trow + (uint32_t)(cbeg + j * 16), r);
          tmem_ld_wait();
          uint8_t* rowp = boxes + j * 2048 + lane * 64;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(rowp + ((q ^ ((lane >> 1) & 3)) << 4)) =
                ok ? make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3])
                   : make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();  // the boxes, before the tensor stores read them
        __syncwarp();
        if (lane == 0) {
          for (int j = 0; j < nbox; ++j)
            tma_store_3d(&tm_part, smem_u32(boxes + j * 2048), cbeg + j * 16,
                         (int32_t)(m0 + lg * 32), split);
          bulk_commit();
          bulk_wait_all();  // the partial tile written (and the boxes read) before the CTA ends
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ------------------------------------------------------- fused dt_proj + scan

struct ScanArgs {
  int64_t L, d, T;
  int R, nslab;
  const bf16* x;
  const bf16* z;
  const bf16* conv_w;
  const bf16* conv_b;
  const float* dt_bias;
  const float* A_log;
  const float* D;
  const float* h0;
  float* hT;
  bf16* y;
  const bf16* hist;
  bf16* final_conv;
  const __half* wdt;  // W_dt in fp16 [d, R]: the compute warps copy its first K slabs to TMEM
  ErrFlags* err;
  // Work schedule (see k_scan_fused).  A pair is one (sequence, 128-channel
  // tile); each pair's sequence is cut into n_parts time parts of whole chunks.
  int64_t B;       // sequences
  const int* cu;   // packed batch: [B + 1] token offsets (else sequence b is tokens b*L ..)
  const int* order;  // packed batch: sequences longest first (claim order), or null
  int n_tiles;     // channel tiles per sequence
  int n_parts;     // time parts per sequence
  int two_pass;    // 0: parts run in a chain; 1: state pass, then output pass
  int* counter;    // next unit to claim
  int* flags;      // [pairs * n_parts]: nonzero once that part's hand-over is written
  float* carry_h;  // [pairs * n_parts, 128, 16]: a part's end state
  float* carry_s;  // [pairs * n_parts, 128]: a part's sum of delta (two-pass)
};

// How the scan kernel cuts the work (host side; also sizes the workspace).
struct ScanPlan {
  int n_parts = 1;
  int two_pass = 0;
};

#ifndef JMIX_SCAN_LEAD
#define JMIX_SCAN_LEAD 0    // 4-warp CTAs whose thread 0 also feeds the ring: 3 CTAs per SM
#endif
#ifndef JMIX_SCAN_CTAS
#define JMIX_SCAN_CTAS (JMIX_SCAN_LEAD ? 3 : 2)
#endif
// CTAs of the scan kernel resident on each of a B200's 148 SMs.
constexpr int kScanCtasPerSm = JMIX_SCAN_CTAS;
constexpr int kScanSlots = kScanCtasPerSm * 148;
// A time part spans at least this many 16-token chunks.
constexpr int kMinPartChunks = 16;

ScanPlan scan_plan(int64_t B, int64_t L, int64_t d) {
  ScanPlan pl;
  const int64_t pairs = B * ((d + kSC - 1) / kSC);
  const int64_t nch = (L + kSQ - 1) / kSQ;
  if (pairs <= 0 || nch <= 0) return pl;
  if (pairs > kScanSlots) {
    // More pairs than CTA slots: parts only even out the last wave.  A part
    // starts from the state of the part before it (a chain), which costs no
    // extra arithmetic; with more pairs than slots a part's predecessor was
    // claimed at least one wave earlier, so chained parts do not wait.  Waves of
    // part-sized units: ceil(pairs*P/slots)/P.
    int64_t best_num = (pairs + kScanSlots - 1) / kScanSlots, best_den = 1;
    for (int P = 2; P <= 8; P *= 2) {
      if (nch < (int64_t)kMinPartChunks * P) break;
      const int64_t num = (pairs * P + kScanSlots - 1) / kScanSlots;
      if (num * best_den < best_num * P) {
        best_num = num;
        best_den = P;
        pl.n_parts = P;
      }
    }
  } else if (pairs < kScanSlots / 2) {
    // Too few pairs for the GPU: a state pass over parts 0..P-2 (from a zero
    // state) runs side by side, then every part produces its outputs from the
    // state that the earlier parts' results fold into.
    int P = 8;
    while (P > 1 && nch < (int64_t)kMinPartChunks * P) P /= 2;
    pl.n_parts = P;
    pl.two_pass = P > 1;
  }
  return pl;
}

// warps 0..3: one channel per thread (its TMEM lane); warp 4: TMA + MMA
constexpr int kProdWarp = 4;
constexpr int kScanThreads = 32 * (kProdWarp + 1);
constexpr int kAllBar = 1;  // named barrier of the four compute warps
// The scan kernel keeps W_dt's first two 64-wide K slabs in TMEM (the MMA's A
// operand may come from there) and only the rest in shared memory, which lets
// three CTAs share an SM.  TMEM per CTA: columns [0, 32) hold the two dt_proj
// accumulators, [64, 128) the W_dt slabs (two fp16 per 32-bit column).
#ifndef JMIX_SCAN_TMEM_SLABS
#define JMIX_SCAN_TMEM_SLABS 2
#endif
#ifndef JMIX_SCAN_STAGES
#define JMIX_SCAN_STAGES 2
#endif
constexpr int kWdtTmemSlabs = JMIX_SCAN_TMEM_SLABS;
constexpr int kScanStages = JMIX_SCAN_STAGES;  // ring of {dt_n, x, z, B/C} stages + accumulators
constexpr int kScanWdtBytes = (kMaxSlabs - kWdtTmemSlabs) * kSC * 128;  // 32 KB
constexpr uint32_t kTmemWdtCol = kScanStages * kSQ <= 64 ? 64 : 128;
constexpr uint32_t kScanTmemNeed = kTmemWdtCol + 32 * kWdtTmemSlabs;
constexpr uint32_t kScanTmemCols = kScanTmemNeed <= 64 ? 64 : kScanTmemNeed <= 128 ? 128
                                   : kScanTmemNeed <= 256 ? 256 : 512;
static_assert(kScanStages * kSQ <= (int)kTmemWdtCol, "accumulators overlap the W_dt columns");
static_assert(kScanCtasPerSm * kScanTmemCols <= 512, "TMEM of the resident CTAs exceeds 512 columns");
constexpr int kDtnStage = kMaxSlabs * kSQ * 128;                  // 16 KB at kSQ = 32 (SW128)
constexpr int kXStage = kSQ * kSC * 2;                            // 8 KB (x or z tile)
constexpr int kBCStage = kSQ * 2 * kN * 4;                        // 4 KB
constexpr int kStageBytes = kDtnStage + 2 * kXStage + kBCStage;   // 36 KB
#ifndef JMIX_SCAN_G
#define JMIX_SCAN_G 8
#endif
constexpr int kG = JMIX_SCAN_G;  // tokens per TMEM load / unrolled group in the scan loop
constexpr int kScanSmem = 1024 + kScanWdtBytes + kScanStages * kStageBytes + 256;
static_assert(kScanCtasPerSm * (kScanSmem + 1024) <= 228 * 1024, "shared memory per SM exceeded");

// softplus(v) = max(v, 0) + log1p(exp(-|v|)): one MUFU ex2, log1p by a
// degree-8 minimax polynomial on the FMA pipe (relative error < 3e-7).
__device__ __forceinline__ float softplus_fast(float v) {
  const float w = ex2_approx(-fabsf(v) * kLog2e);
  float q = poly::L8;
  q = fmaf(q, w, poly::L7);
  q = fmaf(q, w, poly::L6);
  q = fmaf(q, w, poly::L5);
  q = fmaf(q, w, poly::L4);
  q = fmaf(q, w, poly::L3);
  q = fmaf(q, w, poly::L2);
  q = fmaf(q, w, poly::L1);
  q = fmaf(q, w, poly::L0);
  return fmaf(w, q, fmaxf(v, 0.0f));
}


__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// z * sigmoid(z) for the bf16 output gate, sigmoid(z) = (1 + tanh(z/2)) / 2:
// one MUFU op, absolute error of sigmoid ~3e-4, far inside the output's tolerance.
__device__ __forceinline__ float silu_gate(float z) {
  const float hz = 0.5f * z;
  return fmaf(hz, tanh_approx(hz), hz);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Waits (bounded) until *flag is nonzero; one thread calls it.
__device__ __forceinline__ void wait_flag(const int* flag, ErrFlags* err, unsigned site) {
  if (ld_acquire_gpu(flag)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!ld_acquire_gpu(flag)) {
    __nanosleep(64);
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      if (atomicExch(&err->timeout, 1u) == 0u) err->where = site;
      return;
    }
  }
}

// The compute warps' share of one unit: chunks [kb, kb + nch) of the pair's
// sequence.  kOut: produce y (else only the state and the sum of delta).
// Zero-order hold: the factor expm1(delta A) / A that multiplies B u, for a pair
// of states.  x = delta A log2(e) (as passed to ex2), da = 2^x = exp(delta A),
// inv_a = 1 / A.  For |delta A| >= 1/32: (da - 1) / A (relative error below
// 1e-5 with ex2.approx); below: delta (1 + y/2 + y^2/6), y = delta A (the
// series of expm1(y)/y, truncation below 1.3e-6).
__device__ __forceinline__ float2 zoh_factor(float2 x, float2 da, float2 inv_a, float2 dl2) {
  const float2 y = __fmul2_rn(x, make_float2(0.69314718f, 0.69314718f));
  const float2 poly = __ffma2_rn(y, __ffma2_rn(y, make_float2(1.0f / 6.0f, 1.0f / 6.0f),
                                              make_float2(0.5f, 0.5f)),
                                 make_float2(1.0f, 1.0f));
  const float2 small = __fmul2_rn(dl2, poly);
  const float2 big = __fmul2_rn(__fadd2_rn(da, make_float2(-1.0f, -1.0f)), inv_a);
  return make_float2(fabsf(y.x) < 0.03125f ? small.x : big.x,
                     fabsf(y.y) < 0.03125f ? small.y : big.y);
}


#ifndef JMIX_SCAN_SLEEP
#define JMIX_SCAN_SLEEP 256  // ns the scan's producer sleeps between barrier tries (0: spin)
#endif
#ifndef JMIX_SCAN_FULL
#define JMIX_SCAN_FULL 1     // chunks of a full kSQ tokens take a path without per-token checks
#endif

// The per-token terms of one group of kG tokens: delta, the factor of B in the
// update (delta u, or u under zero-order hold), D u and SiLU(z).
struct TokTerms {
  float dl[kG], du[kG], dsk[kG], gz[kG];
};

// Per-token terms of tokens g0t .. g0t + kG - 1 of the current chunk: u =
// SiLU(conv) recomputed in float32 from x (the conv window xw slides over the
// live tokens), delta = softplus(dt_proj accumulator r + bias), and for kOut
// D u and SiLU(z).  Without kOut the live deltas are summed into csum.
template <bool kOut, bool kZoh, bool kFull>
__device__ __forceinline__ void scan_terms(const uint32_t (&r)[kG], const bf16* xs, const bf16* zs,
                                           int g0t, int nt, int cl, float (&xw)[kConv - 1],
                                           const float (&cw)[kConv], float cb, float bias,
                                           float Dc, TokTerms& T, float& csum) {
#pragma unroll
  for (int i = 0; i < kG; ++i) {
    const float xt = bf(xs[(g0t + i) * kSC + cl]);
    float xc = fmaf(cw[0], xw[0], cb);
    xc = fmaf(cw[1], xw[1], xc);
    xc = fmaf(cw[2], xw[2], xc);
    xc = fmaf(cw[3], xt, xc);
    const float uv = silu_newton(xc);
    const bool live = kFull || g0t + i < nt;
    if (live) {
      xw[0] = xw[1];
      xw[1] = xw[2];
      xw[2] = xt;
    }
    T.dl[i] = softplus_fast(__uint_as_float(r[i]) + bias);
    T.du[i] = kZoh ? uv : T.dl[i] * uv;  // zero-order hold: u (the factor is per state)
    if constexpr (kOut) {
      T.dsk[i] = Dc * uv;
      T.gz[i] = silu_gate(bf(zs[(g0t + i) * kSC + cl]));
    } else {
      csum += live ? T.dl[i] : 0.0f;
    }
  }
}

// The 16-state recurrence over tokens g0t .. g0t + kG - 1 (those below nt) of
// the current chunk, with B and C rows from the stage; for kOut, y = (C.h + D u)
// SiLU(z) is stored to yrow (row stride d) when the channel exists.
template <bool kOut, bool kZoh, bool kFull, bool kYS>
__device__ __forceinline__ void scan_recur(const TokTerms& T, const float4* bcs, int g0t, int nt,
                                           float2 (&h)[kN / 2], const float2 (&A2)[kN / 2],
                                           const float2 (&invA)[kN / 2], bf16* yrow,
                                           int64_t tbase, int64_t d, bool cok, bf16* ys_smem,
                                           int cl) {
  static_assert(!kYS || (kFull && kG % 2 == 0), "y through the stage: whole groups of token pairs");
  float yprev = 0.0f;  // (kYS) the even token's y, rounded with the odd one's
#pragma unroll
  for (int i = 0; i < kG; ++i) {
    const int t = g0t + i;
    if (!kFull && t >= nt) break;
    const float2 dl2 = make_float2(T.dl[i], T.dl[i]);
    const float2 du2 = make_float2(T.du[i], T.du[i]);
    float2 acc[4];
#pragma unroll
    for (int q4 = 0; q4 < kN / 4; ++q4) {
      const float4 Bq = bcs[t * 8 + q4];
      float4 Cq;
      if constexpr (kOut) Cq = bcs[t * 8 + 4 + q4];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int q = q4 * 2 + half;
        const float2 Bp = half ? make_float2(Bq.z, Bq.w) : make_float2(Bq.x, Bq.y);
        const float2 x = __fmul2_rn(dl2, A2[q]);
        float2 da;
        da.x = ex2_approx(x.x);
        da.y = ex2_approx(x.y);
        if constexpr (kZoh)
          h[q] = __ffma2_rn(da, h[q],
                            __fmul2_rn(__fmul2_rn(zoh_factor(x, da, invA[q], dl2), du2), Bp));
        else
          h[q] = __ffma2_rn(da, h[q], __fmul2_rn(du2, Bp));
        if constexpr (kOut) {
          // four independent partial sums of C.h (short dependency chains)
          const float2 Cp = half ? make_float2(Cq.z, Cq.w) : make_float2(Cq.x, Cq.y);
          acc[q4] = half ? __ffma2_rn(Cp, h[q], acc[q4]) : __fmul2_rn(Cp, h[q]);
        }
      }
    }
    if constexpr (kOut) {
      const float2 s01 = __fadd2_rn(acc[0], acc[1]);
      const float2 s23 = __fadd2_rn(acc[2], acc[3]);
      const float2 sa = __fadd2_rn(s01, s23);
      const float ys = (sa.x + sa.y) + T.dsk[i];
      if constexpr (kYS) {
        // into the stage's x tile (tokens t - 1 and t's x are already read); two
        // tokens' y are rounded to bf16 by one paired conversion (same bits)
        if (i & 1) {
          const __nv_bfloat162 y2 = __floats2bfloat162_rn(yprev, ys * T.gz[i]);
          ys_smem[(t - 1) * kSC + cl] = y2.x;
          ys_smem[t * kSC + cl] = y2.y;
        } else {
          yprev = ys * T.gz[i];
        }
      } else if (cok)
        yrow[(tbase + t) * d] = __float2bfloat16_rn(ys * T.gz[i]);
    }
  }
}

// The groups of one chunk: tokens 0 .. nt - 1 (kFull: nt == kSQ, so no
// per-token live checks are needed).
template <bool kOut, bool kZoh, bool kFull, bool kYS, class GroupHook>
__device__ __forceinline__ void scan_chunk_body(uint32_t tacc, const bf16* xs, const bf16* zs,
                                                const float4* bcs, int nt, int cl,
                                                float (&xw)[kConv - 1], const float (&cw)[kConv],
                                                float cb, float bias, float Dc,
                                                float2 (&h)[kN / 2], const float2 (&A2)[kN / 2],
                                                const float2 (&invA)[kN / 2], bf16* yrow,
                                                int64_t tbase, int64_t d, bool cok, float& csum,
                                                const GroupHook& ghook) {
#pragma unroll 1
    for (int g0t = 0; g0t < nt; g0t += kG) {
      uint32_t r[kG];
      tmem_ld_cols<kG>(tacc + (uint32_t)g0t, r);
      tmem_ld_wait();
      TokTerms T;
      scan_terms<kOut, kZoh, kFull>(r, xs, zs, g0t, nt, cl, xw, cw, cb, bias, Dc, T, csum);
      scan_recur<kOut, kZoh, kFull, kYS>(T, bcs, g0t, nt, h, A2, invA, yrow, tbase, d, cok,
                                         const_cast<bf16*>(xs), cl);
      ghook();
    }
}

#ifndef JMIX_SCAN_YTMA
#define JMIX_SCAN_YTMA 1    // y of whole chunks leaves through the stage by TMA
#endif
#ifndef JMIX_SCAN_YTMA_PACKED
#define JMIX_SCAN_YTMA_PACKED 1  // ... in packed batches too
#endif
// Whether a chunk of nt tokens of an output unit stores its y tile by TMA from
// the stage (whole chunks: the tile stays inside its sequence), else thread by
// thread.
__device__ __forceinline__ bool y_by_tma(const ScanArgs& a, bool out, int nt) {
  return JMIX_SCAN_YTMA && out && (JMIX_SCAN_YTMA_PACKED || !a.cu) && nt == kSQ;
}

template <bool kOut, bool kZoh, bool kLead, class Hook>
__device__ __forceinline__ void scan_chunks(const Hook& hook, const ScanArgs& a,
                                            const uint8_t* stage0,
                                            uint64_t* full, uint64_t* mma_done, uint64_t* empty,
                                            uint32_t tmem, int warp, int lane, int kg0, int kb,
                                            int nch, int64_t Lb, bool cok, bf16* yrow,
                                            float2 (&h)[kN / 2],
                                            const float2 (&A2)[kN / 2],
                                            const float2 (&invA)[kN / 2], float (&xw)[kConv - 1],
                                            const float (&cw)[kConv], float cb, float bias,
                                            float Dc, float& ssum) {
  const int cl = warp * 32 + lane;
  for (int k = 0; k < nch; ++k) {
    const int kg = kg0 + k;
    const int s = kg % kScanStages;
    const uint32_t ph = (uint32_t)(kg / kScanStages) & 1u;
    if (!mbar_wait(smem_u32(&mma_done[s]), ph, a.err, 25)) break;
    if (!mbar_wait(smem_u32(&full[s]), ph, a.err, 26)) break;
    tc_fence_after();
    const uint8_t* st = stage0 + s * kStageBytes;
    const bf16* xs = reinterpret_cast<const bf16*>(st + kDtnStage);
    const bf16* zs = reinterpret_cast<const bf16*>(st + kDtnStage + kXStage);
    const float4* bcs = reinterpret_cast<const float4*>(st + kDtnStage + 2 * kXStage);
    const int64_t tbase = (int64_t)(kb + k) * kSQ;
    const int nt = (int)((Lb - tbase) < kSQ ? (Lb - tbase) : kSQ);
    const uint32_t tacc = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(s * kSQ);
    float csum = 0.0f;
    // whole chunks of fixed-length sequences leave y in the stage; the producer
    // stores the [32 x 128] y tile by TMA (partial chunks store y directly)
    const bool ytile = y_by_tma(a, kOut && !kLead, nt);
    auto ghook = [&]() { hook(k, false); };
    if (ytile)
      scan_chunk_body<kOut, kZoh, true, true>(tacc, xs, zs, bcs, nt, cl, xw, cw, cb, bias, Dc, h,
                                              A2, invA, yrow, tbase, a.d, cok, csum, ghook);
    else if (JMIX_SCAN_FULL && nt == kSQ)
      scan_chunk_body<kOut, kZoh, true, false>(tacc, xs, zs, bcs, nt, cl, xw, cw, cb, bias, Dc, h,
                                               A2, invA, yrow, tbase, a.d, cok, csum, ghook);
    else
      scan_chunk_body<kOut, kZoh, false, false>(tacc, xs, zs, bcs, nt, cl, xw, cw, cb, bias, Dc, h,
                                                A2, invA, yrow, tbase, a.d, cok, csum, ghook);
    if constexpr (!kOut) ssum += csum;
    if (ytile) fence_proxy_async_smem();  // y in the stage, before the TMA store reads it
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    hook(k, true);
  }
}

// Claim order of a packed batch's sequences: longest first (ties by index), so
// that the long sequences, which set the scan's critical path, start first.
// One CTA; rank of b = number of sequences that come before it.  Lengths of a
// broken cu are clamped to [0, T] here (the scan kernel reports it).
__global__ void __launch_bounds__(1024) k_order_by_length(const int* __restrict__ cu, int B,
                                                         int T, int* __restrict__ order) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    auto len = [&](int i) {
      const int v = __ldg(cu + i + 1) - __ldg(cu + i);
      return v < 0 ? 0 : (v > T ? T : v);
    };
    const int lb = len(b);
    int rank = 0;
    for (int i = 0; i < B; ++i) {
      const int li = len(i);
      rank += (li > lb) || (li == lb && i < b);
    }
    order[rank] = b;  // ranks are a permutation of 0 .. B-1
  }
}

// Fused dt_proj (tcgen05, accumulator in TMEM) + softplus + selective scan +
// D skip + SiLU(z) gate, with the causal conv + SiLU recomputed in fp32 from x.
//
// Persistent CTAs (two per SM) claim units from a counter.  A unit is one
// time part of one pair (sequence, 128-channel tile); warp 4 streams its
// chunks (dt_n, x, z, B/C rows) by TMA and issues the dt_proj MMAs, warps 0..3
// run the recurrence with one channel per thread.
//   chain (two_pass = 0): parts of a pair run in order, each starting from the
//     end state that the part before it hands over.
//   two-pass: state units for parts 0..P-2 run the recurrence from a zero
//     state (part 0: from the initial state) and record the end state and the
//     sum S of delta; the output unit of part p starts from the fold of parts
//     0..p-1: h <- exp(A S_q) h + h_end_q, since the state map of a part is
//     h -> exp(A S) h + h_end(zero start), A being constant over time.
// Every unit that waits waits only for units that come before it in claim
// order, and a claimed unit is running or queued behind one with a smaller
// index on its CTA, so every wait ends; each is still bounded (2 s).
// kLead: no producer warp; thread 0 issues the ring's TMA loads and the dt_proj
// MMAs between its own groups of tokens (4 warps per CTA, 3 CTAs per SM).
template <bool kZoh, bool kLead>  // B by zero-order hold (else delta B)
__global__ void __launch_bounds__(kLead ? 128 : kScanThreads, kScanCtasPerSm)
    k_scan_fused(const __grid_constant__ CUtensorMap tm_wdt,
                 const __grid_constant__ CUtensorMap tm_dtn,
                 const __grid_constant__ CUtensorMap tm_bc, const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_y,
                 const ScanArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // (offset arithmetic on the shared array keeps its address space known, so
  // accesses through these pointers compile to shared-memory loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* wdt_s = smem;                  // W_dt K slabs 2.. : [128 ch x 64] each (SW128)
  uint8_t* stage0 = smem + kScanWdtBytes;  // 2 x {dt_n (SW128), x tile, z tile, B/C rows}
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage0 + kScanStages * kStageBytes);
  uint64_t* full = bars;                         // [stages] stage landed
  uint64_t* mma_done = bars + kScanStages;       // [stages] dt_proj accumulator ready
  uint64_t* empty = bars + 2 * kScanStages;      // [stages] compute warps done with the slot
  uint64_t* wfull = bars + 3 * kScanStages;      // W_dt slabs in shared memory landed
  uint64_t* wready = wfull + 1;  // W_dt slabs in TMEM written (one arrive per compute warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfull + 2);
  volatile int* unit_slot = reinterpret_cast<volatile int*>(wfull + 3);  // [2] claimed units
  const int nslab_t = a.nslab < kWdtTmemSlabs ? a.nslab : kWdtTmemSlabs;  // slabs in TMEM

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = a.n_tiles * (int)a.B;
  const int P = a.n_parts;
  const int n_state = a.two_pass ? pairs * (P - 1) : 0;  // state units come first
  const int n_units = n_state + pairs * P;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&mma_done[s]), 1);
      mbar_init(smem_u32(&empty[s]), kProdWarp);  // one arrive per compute warp
    }
    mbar_init(smem_u32(wfull), 1);
    mbar_init(smem_u32(wready), 4);
    fence_mbar_init();
  }
  constexpr int kAllocWarp = kLead ? 0 : kProdWarp;
  constexpr int kFeedThread = kLead ? 0 : 32 * kProdWarp;  // claims units, feeds the ring
  if (warp == kAllocWarp) {
    tmem_alloc(smem_u32(tmem_slot), kScanTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();    // dt_n, B/C and the fp16 W_dt come from the kernels before it
  // claim the first unit only now: a CTA that waited in tcgen05.alloc (more
  // CTAs resident than TMEM for) holds no unit that another CTA could wait on
  if (threadIdx.x == 0) unit_slot[0] = atomicAdd(a.counter, 1);
  __syncthreads();

  int kg0 = 0;    // chunks this CTA has run before the current unit (mbarrier phases)
  int nw = 0;     // W_dt tiles this CTA has loaded (wfull phase)
  for (int it = 0;; ++it) {
    const int unit = unit_slot[it & 1];
    if (unit >= n_units) break;
    // claim the next unit early, so that its number is ready when this one ends
    if (threadIdx.x == kFeedThread)
      unit_slot[(it + 1) & 1] = *(volatile unsigned*)&a.err->timeout ? n_units
                                                                      : atomicAdd(a.counter, 1);
    const bool out = unit >= n_state;
    const int uu = out ? unit - n_state : unit;
    const int part = uu / pairs;
    const int pair = uu - part * pairs;
    const int64_t bq = pair / a.n_tiles;
    const int tile = pair - (int)bq * a.n_tiles;
    const int64_t b = a.order ? a.order[bq] : bq;  // packed: longest sequences are claimed first
    const int64_t c0 = (int64_t)tile * kSC;
    // the sequence's first token and length (packed batch: from cu, checked here;
    // a broken cu is reported and the sequence treated as empty)
    int64_t g0 = b * a.L, Lb = a.L;
    if (a.cu) {
      const int s0 = a.cu[b], s1 = a.cu[b + 1];
      if (s0 < 0 || s1 < s0 || s1 > a.T || (b == 0 && s0 != 0) || (b == a.B - 1 && s1 != a.T)) {
        if (threadIdx.x == 0) atomicExch(&a.err->bad_input, 1u);
        g0 = 0;
        Lb = 0;
      } else {
        g0 = s0;
        Lb = s1 - s0;
      }
    }
    const int nch_all = (int)((Lb + kSQ - 1) / kSQ);
    const int kb = (int)((int64_t)nch_all * part / P);
    const int nch = (int)((int64_t)nch_all * (part + 1) / P) - kb;
    const int64_t hslot = (int64_t)pair * P + part;  // this part's hand-over slot

    // ---- feeding the ring (the producer warp's lane 0, or thread 0 with kLead):
    // its waits last about a chunk of the compute warps' work, so the producer
    // sleeps between tries and its scheduler's slots go to the compute warps
        auto kWait = [](uint32_t bar, uint32_t par, ErrFlags* e, unsigned site) {
          return JMIX_SCAN_SLEEP > 0 && !kLead
                     ? mbar_wait_sleep(bar, par, e, site, JMIX_SCAN_SLEEP)
                     : mbar_wait(bar, par, e, site);
        };
        const uint32_t wb = smem_u32(wfull);
        auto issue_wdt = [&]() {  // W_dt K slabs past the TMEM ones, into shared memory
          if (a.nslab > nslab_t) {
            mbar_arrive_expect_tx(wb, (uint32_t)((a.nslab - nslab_t) * kSC * 128));
            for (int j = nslab_t; j < a.nslab; ++j)
              tma_load_2d(smem_u32(wdt_s + (j - nslab_t) * kSC * 128), &tm_wdt, wb, j * 64,
                          (int32_t)c0);
          }
        };
        const uint32_t stage_tx =
            (uint32_t)(a.nslab * kSQ * 128 + (out ? 2 : 1) * kXStage + kBCStage);
        auto issue_stage = [&](int k) {  // k: chunk of this unit
          const int s = (kg0 + k) % kScanStages;
          uint8_t* st = stage0 + s * kStageBytes;
          const uint32_t fb = smem_u32(&full[s]);
          const int32_t row = (int32_t)(g0 + (int64_t)(kb + k) * kSQ);
          mbar_arrive_expect_tx(fb, stage_tx);
          for (int j = 0; j < a.nslab; ++j)
            tma_load_2d(smem_u32(st + j * kSQ * 128), &tm_dtn, fb, j * 64, row);
          tma_load_2d(smem_u32(st + kDtnStage), &tm_x, fb, (int32_t)c0, row);
          if (out) tma_load_2d(smem_u32(st + kDtnStage + kXStage), &tm_z, fb, (int32_t)c0, row);
          tma_load_2d(smem_u32(st + kDtnStage + 2 * kXStage), &tm_bc, fb, 0, row);
        };
        // y tile of chunk k (whole chunks): the compute warps left it in the
        // stage's x tile; one TMA store per chunk (y is [B, L, d], or [1, T, d]
        // for a packed batch, whose sequence starts at token g0)
        auto store_y = [&](int k) -> bool {
          if (!y_by_tma(a, out, (int)((Lb - (int64_t)(kb + k) * kSQ) < kSQ
                                          ? (Lb - (int64_t)(kb + k) * kSQ) : kSQ)))
            return false;
          const int s = (kg0 + k) % kScanStages;
          tma_store_3d(&tm_y, smem_u32(stage0 + s * kStageBytes + kDtnStage), (int32_t)c0,
                       (int32_t)((a.cu ? g0 : 0) + (int64_t)(kb + k) * kSQ),
                       (int32_t)(a.cu ? 0 : b));
          bulk_commit();
          return true;
        };
        const uint32_t idesc = idesc_f16_f32(kSC, kSQ);
        auto issue_mma = [&](int k) -> bool {
          const int kg = kg0 + k;
          const int s = kg % kScanStages;
          if (!kWait(smem_u32(&full[s]), (uint32_t)(kg / kScanStages) & 1u, a.err, 22))
            return false;
          tc_fence_after();
          const uint32_t wbase = smem_u32(wdt_s), db = smem_u32(stage0 + s * kStageBytes);
          const uint32_t d_tmem = tmem + (uint32_t)(s * kSQ);
          for (int j = 0; j < a.nslab; ++j)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bdesc = sw128_kmajor_desc(db + j * kSQ * 128 + kk * 32);
              const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
              if (j < nslab_t)  // A: 16 K values = 8 TMEM columns per step
                umma_f16_ts(d_tmem, tmem + kTmemWdtCol + (uint32_t)(j * 32 + kk * 8), bdesc, idesc,
                            acc);
              else
                umma_f16(d_tmem, sw128_kmajor_desc(wbase + (j - nslab_t) * kSC * 128 + kk * 32),
                         bdesc, idesc, acc);
            }
          umma_commit(smem_u32(&mma_done[s]));
          return true;
        };
    if (!kLead && warp == kProdWarp) {
      if (lane == 0 && nch > 0) {
        issue_wdt();
        // Every stage and accumulator is free here: the previous unit ended
        // with every compute warp past its last chunk (CTA barrier below).
        for (int k = 0; k < kScanStages && k < nch; ++k) issue_stage(k);
        bool ok = a.nslab <= nslab_t || kWait(wb, (uint32_t)nw & 1u, a.err, 21);
        if (ok) ok = kWait(smem_u32(wready), (uint32_t)nw & 1u, a.err, 27);
        if (ok) tc_fence_after();
        if (ok) ok = issue_mma(0);
        // chunk j's slot (stage + accumulator) is reused by chunk j + stages, once
        // the compute warps have released chunk j (empty)
        for (int k = 0; ok && k < nch; ++k) {
          const int kg = kg0 + k;
          if (k + 1 < nch) {
            const int j = kg + 1 - kScanStages;  // last chunk in MMA k+1's accumulator
            if (j >= kg0 && !kWait(smem_u32(&empty[j % kScanStages]),
                                   (uint32_t)(j / kScanStages) & 1u, a.err, 23))
              break;
            if (!issue_mma(k + 1)) break;
          }
          if (k + kScanStages < nch) {
            if (!kWait(smem_u32(&empty[kg % kScanStages]), (uint32_t)(kg / kScanStages) & 1u,
                           a.err, 24))
              break;
            if (store_y(k)) bulk_wait_read<0>();  // the stage is reloaded right after
            issue_stage(k + kScanStages);
          }
        }
        // the y tiles of the last chunks (no reload follows them)
        for (int k = nch > kScanStages ? nch - kScanStages : 0; ok && k < nch; ++k) {
          const int kg = kg0 + k;
          if (!kWait(smem_u32(&empty[kg % kScanStages]), (uint32_t)(kg / kScanStages) & 1u,
                     a.err, 29))
            break;
          store_y(k);
        }
        bulk_wait_read<0>();  // the next unit reuses every stage
      }
    } else {
      // compute warps: thread = channel c0 + 32*warp + lane = TMEM lane
      const int cl = warp * 32 + lane;
      const int64_t c = c0 + cl;
      const bool cok = c < a.d;
      bool lead_ok = true;  // kLead, thread 0: no bounded wait has given up
      if (kLead && threadIdx.x == 0 && nch > 0) {
        // every stage and accumulator is free at a unit's start (CTA barrier below)
        issue_wdt();
        for (int k = 0; k < kScanStages && k < nch; ++k) issue_stage(k);
      }
      if (nch > 0) {
        // this channel's W_dt row, K slabs 0..nslab_t-1, into its TMEM lane
        // (zeros past R and past d, matching the zero fill of the dt_n tiles)
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16) + kTmemWdtCol;
        // a 64-wide K slab is 32 columns: nslab_t * 2 steps of 16 columns stay
        // inside [kTmemWdtCol, kTmemWdtCol + 64) of the 128-column allocation
        for (int q = 0; q < nslab_t * 2; ++q) {  // 16 columns = 32 K values per step
          uint32_t v[16];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = q * 32 + e * 8;
            uint4 w8 = make_uint4(0u, 0u, 0u, 0u);
            if (cok && k < a.R) w8 = __ldg(reinterpret_cast<const uint4*>(a.wdt + c * a.R + k));
            v[4 * e] = w8.x;
            v[4 * e + 1] = w8.y;
            v[4 * e + 2] = w8.z;
            v[4 * e + 3] = w8.w;
          }
          tmem_st16(trow + (uint32_t)(q * 16), v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(wready));
      }
      if (kLead && threadIdx.x == 0 && nch > 0) {  // the first chunk's dt_proj
        lead_ok = a.nslab <= nslab_t || kWait(wb, (uint32_t)nw & 1u, a.err, 21);
        if (lead_ok) lead_ok = kWait(smem_u32(wready), (uint32_t)nw & 1u, a.err, 27);
        if (lead_ok) tc_fence_after();
        if (lead_ok) lead_ok = issue_mma(0);
      }
      // kLead, thread 0: feeds chunk k + 1 while the warps run chunk k.  Its stage
      // and accumulator were chunk k - 1's, so the TMA goes out once every warp
      // is done with chunk k - 1 and the MMA once the TMA has landed; between
      // groups of tokens only non-blocking tests, at the chunk's end waits.
      bool tma_next = true, mma_next = false;  // for chunk 1: its TMA went out above
      auto hook = [&](int k, bool block) {
        if (!kLead || threadIdx.x != 0 || !lead_ok || k + 1 >= nch) return;
        const int kg = kg0 + k;
        if (!tma_next) {
          const int j = kg - 1;
          const uint32_t eb = smem_u32(&empty[j % kScanStages]);
          const uint32_t ep = (uint32_t)(j / kScanStages) & 1u;
          if (!(block ? (lead_ok = kWait(eb, ep, a.err, 23)) : mbar_test_wait(eb, ep))) return;
          issue_stage(k + 1);
          tma_next = true;
        }
        if (!mma_next) {
          const int kn = kg + 1;
          const uint32_t fb = smem_u32(&full[kn % kScanStages]);
          if (!block && !mbar_test_wait(fb, (uint32_t)(kn / kScanStages) & 1u)) return;
          if (!(lead_ok = issue_mma(k + 1))) return;
          mma_next = true;
        }
        if (block) tma_next = mma_next = false;  // chunk k + 2 is next
      };
      // a unit that starts from earlier parts waits (bounded) for their hand-over
      const int n_wait = part == 0 ? 0 : (a.two_pass ? (out ? part : 0) : 1);
      if (n_wait > 0) {
        if (threadIdx.x == 0) {
          for (int q = part - n_wait; q < part; ++q)
            wait_flag(a.flags + (int64_t)pair * P + q, a.err, 28);
          __threadfence();
        }
        named_bar_sync(kAllBar, 32 * kProdWarp);
      }
      float2 A2[kN / 2], h[kN / 2], invA[kN / 2];
#pragma unroll
      for (int q = 0; q < kN / 2; ++q) {
        const int n = 2 * q;
        A2[q].x = cok ? -expf(a.A_log[c * kN + n]) * kLog2e : 0.0f;
        A2[q].y = cok ? -expf(a.A_log[c * kN + n + 1]) * kLog2e : 0.0f;
        // 1 / A = -exp(-A_log) (zero-order hold only)
        invA[q] = cok ? make_float2(-expf(-a.A_log[c * kN + n]), -expf(-a.A_log[c * kN + n + 1]))
                      : make_float2(0.0f, 0.0f);
        h[q] = make_float2(0.0f, 0.0f);
        if (part == 0 && cok && a.h0) {
          h[q].x = a.h0[(b * a.d + c) * kN + n];
          h[q].y = a.h0[(b * a.d + c) * kN + n + 1];
        }
      }
      if (n_wait > 0) {
        const float* ch = a.carry_h + ((int64_t)pair * P + (part - n_wait)) * kSC * kN + cl * kN;
#pragma unroll
        for (int q = 0; q < kN / 2; ++q) h[q] = __ldcg(reinterpret_cast<const float2*>(ch) + q);
        // two-pass: fold in parts 1..p-1 (h <- exp2(A2 S) h + h_end)
        for (int qp = part - n_wait + 1; qp < part; ++qp) {
          const int64_t sl = (int64_t)pair * P + qp;
          const float S = __ldcg(a.carry_s + sl * kSC + cl);
          const float2* he = reinterpret_cast<const float2*>(a.carry_h + sl * kSC * kN + cl * kN);
#pragma unroll
          for (int q = 0; q < kN / 2; ++q) {
            const float2 e = __ldcg(he + q);
            h[q].x = fmaf(ex2_approx(A2[q].x * S), h[q].x, e.x);
            h[q].y = fmaf(ex2_approx(A2[q].y * S), h[q].y, e.y);
          }
        }
      }
      const float bias = cok ? a.dt_bias[c] : 0.0f;
      const float Dc = cok ? a.D[c] : 0.0f;
      float cw[kConv], xw[kConv - 1];
#pragma unroll
      for (int k = 0; k < kConv; ++k) cw[k] = cok ? bf(a.conv_w[c * kConv + k]) : 0.0f;
      const float cb = cok ? bf(a.conv_b[c]) : 0.0f;
      // conv window: the d_conv-1 inputs before the unit's first token
      const int64_t t0 = (int64_t)kb * kSQ;
#pragma unroll
      for (int k = 0; k < kConv - 1; ++k) {
        const int64_t t = t0 - (kConv - 1) + k;
        xw[k] = !cok ? 0.0f
                : t >= 0 ? bf(a.x[(g0 + t) * a.d + c])
                : a.hist ? bf(a.hist[(b * a.d + c) * (kConv - 1) + (kConv - 1 + t)])
                         : 0.0f;
      }
      float ssum = 0.0f;
      if (out)
        scan_chunks<true, kZoh, kLead>(hook, a, stage0, full, mma_done, empty, tmem, warp, lane,
                                       kg0, kb, nch,
                                Lb, cok, a.y + g0 * a.d + c, h, A2, invA, xw, cw, cb, bias, Dc,
                                ssum);
      else
        scan_chunks<false, kZoh, kLead>(hook, a, stage0, full, mma_done, empty, tmem, warp, lane,
                                        kg0, kb, nch,
                                 Lb, cok, nullptr, h, A2, invA, xw, cw, cb, bias, Dc, ssum);
      if (part + 1 < P && (!out || !a.two_pass)) {
        // hand the end state (and, two-pass, the sum of delta) to later parts
        float* ch = a.carry_h + hslot * kSC * kN + cl * kN;
#pragma unroll
        for (int q = 0; q < kN / 2; ++q) reinterpret_cast<float2*>(ch)[q] = h[q];
        if (!out) a.carry_s[hslot * kSC + cl] = ssum;
        __threadfence();
        named_bar_sync(kAllBar, 32 * kProdWarp);
        if (threadIdx.x == 0) st_release_gpu(a.flags + hslot, 1);
      } else if (out && part + 1 == P && cok) {
#pragma unroll
        for (int q = 0; q < kN / 2; ++q) {
          a.hT[(b * a.d + c) * kN + 2 * q] = h[q].x;
          a.hT[(b * a.d + c) * kN + 2 * q + 1] = h[q].y;
        }
        // the conv window now holds the last d_conv-1 inputs (exact bf16 values)
        if (a.final_conv) {
#pragma unroll
          for (int k = 0; k < kConv - 1; ++k)
            a.final_conv[(b * a.d + c) * (kConv - 1) + k] = __float2bfloat16_rn(xw[k]);
        }
      }
    }
    kg0 += nch;
    nw += nch > 0 ? 1 : 0;
    __syncthreads();
    // stop claiming work once any wait has given up
    if (threadIdx.x == kFeedThread && *(volatile unsigned*)&a.err->timeout)
      unit_slot[(it + 1) & 1] = n_units;
    __syncthreads();
  }
  if (!kLead && threadIdx.x == kFeedThread) bulk_wait_all();  // the y tile stores completed
  tc_fence_before();
  __syncthreads();
  if (warp == kAllocWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kScanTmemCols);
  }
}

// ------------------------------------------------------------- decode step
// One token per row.  The work is B x (d / 128) pairs (row, 128-channel tile);
// each of the persistent CTAs (two per SM) takes a contiguous share of them in
// tile-major order (equal once each change of tile is counted as
// kDecSwitchRows rows), so it changes channel tile at most a few times and
// keeps that tile's W_dt in TMEM (the dt_proj MMA's A operand).
//   warp 5: per group of kDB = 16 rows of a tile, TMA-loads the rows' dt_n
//     (SW128, the MMA's B operand) and B/C rows into one of two buffers and
//     issues dt_proj into one of two TMEM accumulators (lane = channel,
//     column = row).
//   warp 4: per row, loads the row's SSM-state tile ([128 channels x 16] fp32,
//     8 KB, by a 2-D TMA with 64-byte swizzle), conv-state tile (768 B), x and
//     z (256 B each) into a ring of kDecStages stages, kDecStages rows ahead.
//   warps 0..3 (thread = channel): per row, read the stage into registers and
//     release it, then conv + SiLU, softplus, the 16-state update, the gate,
//     and store y, the state and the shifted conv state straight to global.
// The state read and write (64 B each per row and channel) is the HBM traffic
// that bounds the step.  Rows whose state slot is outside the pool (indexed
// step) are reported and skipped: nothing is loaded from or stored to a slot
// outside the pool.
#ifndef JMIX_DEC_SWITCH_ROWS
#define JMIX_DEC_SWITCH_ROWS 12
#endif
constexpr int kDecSwitchRows = JMIX_DEC_SWITCH_ROWS;      // a W_dt reload, in rows of work
constexpr int kDB = 16;                                   // rows per dt_proj MMA (N)
constexpr int kDecThreads = 192;
constexpr int kDecStages = 8;
constexpr int kDecState = kSC * kN * 4;                   // 8 KB state tile
constexpr int kDecConv = kSC * (kConv - 1) * 2;           // 768 B conv-state tile
constexpr int kDecRow = kSC * 2;                          // 256 B of x or z
constexpr int kDecStage = 10240;                          // state | conv | x | z, 1 KB aligned
static_assert(kDecState + kDecConv + 2 * kDecRow <= kDecStage, "decode stage overflow");
constexpr int kDecDtn = kMaxSlabs * kDB * 128;            // 8 KB (SW128 slabs)
constexpr int kDecBC = kDB * 2 * kN * 4;                  // 2 KB
// A warp's write-back scratch: 32 state rows (2 KB, 64-byte swizzle) and their
// conv states (192 B), 512-byte aligned (the swizzle pattern's period).
constexpr int kDecWb = 2560;
static_assert(kDecWb >= 32 * kN * 4 + 32 * (kConv - 1) * 2 && kDecWb % 512 == 0, "scratch");
constexpr int kDecSmem =
    1024 + kDecStages * kDecStage + 2 * kDecDtn + 2 * kDecBC + 4 * kDecWb + 256;
static_assert(2 * (kDecSmem + 1024) <= 228 * 1024, "two decode CTAs per SM");
constexpr uint32_t kDecTmemCols = 256;                    // W_dt [0, 128) | acc 128 + 16 b
constexpr uint32_t kDecAccCol = 128;

struct DecArgs {
  int64_t B, d;
  int nslab, R;
  int64_t pairs;       // B * tiles
  int n_tiles;
  const bf16* x;
  const bf16* z;
  const bf16* conv_w;
  const bf16* conv_b;
  const float* dt_bias;
  const float* A_log;
  const float* D;
  const uint16_t* wdt;  // W_dt [d, R]: the prepared fp16 copy, or (wdt_bf16) the bf16 input,
  int wdt_bf16;         // which is rounded to fp16 on its way into TMEM
  bf16* conv_state;    // [B, d, 3] in/out (indexed: [n_slots, d, 3])
  float* ssm_state;    // [B, d, 16] in/out (indexed: [n_slots, d, 16])
  bf16* y;
  ErrFlags* err;
  const int* sidx;     // indexed step: state slot of each row, or null (slot = row)
  int64_t n_slots;
};

// State slot of row b, or -1 when it is outside the pool.
__device__ __forceinline__ int64_t dec_slot(const DecArgs& a, int64_t b) {
  if (!a.sidx) return b;
  const int64_t sl = __ldg(a.sidx + b);
  return (sl >= 0 && sl < a.n_slots) ? sl : -1;
}

template <bool kZoh>  // B by zero-order hold (else delta B)
__global__ void __launch_bounds__(kDecThreads, 2)
    k_decode_scan(const __grid_constant__ CUtensorMap tm_state,
                  const __grid_constant__ CUtensorMap tm_state_wb,
                  const __grid_constant__ CUtensorMap tm_dtn,
                  const __grid_constant__ CUtensorMap tm_bc,
                  const __grid_constant__ CUtensorMap tm_wdt, const DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // (offset arithmetic on the shared array keeps its address space known, so
  // accesses through these pointers compile to shared-memory loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;                                  // kDecStages x kDecStage
  uint8_t* dtn_s = stages + kDecStages * kDecStage;        // 2 x kDecDtn
  uint8_t* bc_s = dtn_s + 2 * kDecDtn;                     // 2 x kDecBC
  uint8_t* wb_s = bc_s + 2 * kDecBC;                       // 4 x kDecWb
  uint64_t* bars = reinterpret_cast<uint64_t*>(wb_s + 4 * kDecWb);
  uint64_t* full = bars;                                   // [stages] row landed
  uint64_t* empty = bars + kDecStages;                     // [stages] row read (4 warps)
  uint64_t* gfull = bars + 2 * kDecStages;                 // [2] dt_n + B/C landed
  uint64_t* mma_done = gfull + 2;                          // [2] accumulator ready
  uint64_t* acc_free = mma_done + 2;                       // [2] group done (4 warps)
  uint64_t* wready = acc_free + 2;                         // W_dt of a new tile in TMEM
  uint64_t* wfull = wready + 1;                            // the first tile's W_dt in the ring
  uint64_t* wcopied = wready + 2;                          // ... and out of it (4 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wready + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's pairs [p0, p1), tile-major: pair p = (tile p / B, row p % B).
  // A CTA whose range crosses into another tile reloads W_dt on the way (its
  // first tile's load overlaps the wait for the norms), which costs about
  // kDecSwitchRows rows of work: the ranges are equal shares of a virtual
  // sequence in which each tile starts with that many units of no rows.
  constexpr int64_t P = kDecSwitchRows;
  const int64_t Bv = a.B + P;
  const int64_t V = (int64_t)a.n_tiles * Bv;
  auto pair_at = [&](int64_t v) {
    const int64_t t = v / Bv, r = v - t * Bv - P;
    return t * a.B + (r < 0 ? 0 : r);
  };
  const int64_t p0 = pair_at(V * blockIdx.x / gridDim.x);
  const int64_t p1 = pair_at(V * (blockIdx.x + 1) / gridDim.x);
  const int64_t ngrp = (a.B + kDB - 1) / kDB;  // row groups per tile
  // groups this CTA touches: g = tile * ngrp + row / kDB
  auto grp_of = [&](int64_t p) { return (p / a.B) * ngrp + (p % a.B) / kDB; };
  const int64_t g0 = p0 < p1 ? grp_of(p0) : 0;
  const int64_t g1 = p0 < p1 ? grp_of(p1 - 1) + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 4);  // one arrive per compute warp, once it read the stage
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&gfull[b]), 1);
      mbar_init(smem_u32(&mma_done[b]), 1);
      mbar_init(smem_u32(&acc_free[b]), 4);
    }
    mbar_init(smem_u32(wready), 4);
    mbar_init(smem_u32(wfull), 1);
    mbar_init(smem_u32(wcopied), 4);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), kDecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---- row streamer: the inputs do not depend on earlier kernels of the
    // step (the conv kernel only reads the conv states), so it starts at once
    if (lane == 0) {
      prefetch_tmap(&tm_state);
      const uint64_t evict_first = l2_evict_first_policy();
      int64_t pend_s = p1;  // the rows this streamer loads: [p0, pend_s)
      if (p0 < p1) {
        // the first tile's W_dt rows come through the ring (one 16 KB box per 64
        // K values, 128-byte swizzle: the compute threads' row reads are free of
        // bank conflicts); the state rows follow once the compute warps have
        // moved them into TMEM
        prefetch_tmap(&tm_wdt);
        const uint32_t wf = smem_u32(wfull);
        mbar_arrive_expect_tx(wf, (uint32_t)(a.nslab * kSC * 128));
        for (int j = 0; j < a.nslab; ++j)
          tma_load_2d(smem_u32(stages + j * kSC * 128), &tm_wdt, wf, j * 64,
                      (int32_t)((p0 / a.B) * kSC));
        if (!mbar_wait(smem_u32(wcopied), 0u, a.err, 47)) pend_s = p0;  // (reported; no rows)
      }
      // (tile, row) of pair p, advanced by one row per pair (no divisions in the loop)
      int64_t tile = p0 / a.B, b = p0 - tile * a.B;
      for (int64_t p = p0, i = 0; p < pend_s; ++p, ++i, ++b) {
        if (b == a.B) {
          b = 0;
          ++tile;
        }
        const int s = (int)(i % kDecStages);
        if (i >= kDecStages &&
            !mbar_wait(smem_u32(&empty[s]), (uint32_t)((i / kDecStages) - 1) & 1u, a.err, 41))
          break;
        const int64_t c0 = tile * kSC;
        const int64_t sl = dec_slot(a, b);
        // channels of this tile that exist (a multiple of 8): the 1-D copies
        // stop there, so none reads past the end of its buffer
        const int64_t nc = (a.d - c0) < kSC ? (a.d - c0) : kSC;
        const uint32_t conv_bytes = (uint32_t)(nc * (kConv - 1) * 2), row_bytes = (uint32_t)(nc * 2);
        uint8_t* st = stages + s * kDecStage;
        const uint32_t fb = smem_u32(&full[s]);
        if (sl >= 0) {
          mbar_arrive_expect_tx(fb, (uint32_t)kDecState + conv_bytes + 2 * row_bytes);
          // (the state is streamed through once a step: evict-first in L2, for
          // the load and for the tensor store that writes it back)
          tma_load_3d(smem_u32(st), &tm_state, fb, 0, (int32_t)c0, (int32_t)sl, evict_first);
          bulk_load(smem_u32(st + kDecState), a.conv_state + (sl * a.d + c0) * (kConv - 1),
                    conv_bytes, fb);
        } else {
          mbar_arrive_expect_tx(fb, 2 * row_bytes);
        }
        bulk_load(smem_u32(st + kDecState + kDecConv), a.x + b * a.d + c0, row_bytes, fb);
        bulk_load(smem_u32(st + kDecState + kDecConv + kDecRow), a.z + b * a.d + c0, row_bytes,
                  fb);
      }
    }
  } else if (warp == 5) {
    // ---- dt_proj issuer: dt_n and B/C come from the norms kernel
    if (lane == 0) {
      prefetch_tmap(&tm_dtn);
      prefetch_tmap(&tm_bc);
      grid_dep_wait();
      const uint32_t idesc = idesc_f16_f32(kSC, kDB);
      int64_t cur_tile = -1;
      int ntile = 0;
      for (int64_t g = g0, k = 0; g < g1; ++g, ++k) {
        const int bsel = (int)(k & 1);
        if (k >= 2 &&
            !mbar_wait(smem_u32(&acc_free[bsel]), (uint32_t)((k >> 1) - 1) & 1u, a.err, 42))
          break;
        const int64_t tile = g / ngrp, r0 = (g % ngrp) * kDB;
        const uint32_t gb = smem_u32(&gfull[bsel]);
        uint8_t* dtb = dtn_s + bsel * kDecDtn;
        mbar_arrive_expect_tx(gb, (uint32_t)(a.nslab * kDB * 128 + kDecBC));
        for (int j = 0; j < a.nslab; ++j)
          tma_load_2d(smem_u32(dtb + j * kDB * 128), &tm_dtn, gb, j * 64, (int32_t)r0);
        tma_load_2d(smem_u32(bc_s + bsel * kDecBC), &tm_bc, gb, 0, (int32_t)r0);
        if (!mbar_wait(gb, (uint32_t)(k >> 1) & 1u, a.err, 43)) break;
        if (tile != cur_tile) {  // the compute warps put this tile's W_dt into TMEM
          if (!mbar_wait(smem_u32(wready), (uint32_t)ntile & 1u, a.err, 44)) break;
          cur_tile = tile;
          ++ntile;
        }
        tc_fence_after();
        const uint32_t db = smem_u32(dtb);
        const uint32_t d_tmem = tmem + kDecAccCol + (uint32_t)(bsel * kDB);
        for (int j = 0; j < a.nslab; ++j)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_ts(d_tmem, tmem + (uint32_t)(j * 32 + kk * 8),
                        sw128_kmajor_desc(db + j * kDB * 128 + kk * 32), idesc,
                        (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(smem_u32(&mma_done[bsel]));
      }
    }
  } else {
    // ---- compute warps: thread = channel c0 + cl of the current tile
    const int cl = warp * 32 + lane;
    int64_t cur_tile = -1;
    bool cok = false;
    int64_t c = 0;
    float2 A2[kN / 2];
    float bias = 0.f, Dc = 0.f, cb = 0.f, cw[kConv] = {0.f, 0.f, 0.f, 0.f};
    // 8 W_dt values (bf16, or the prepared fp16) as fp16 pairs
    auto to_half8 = [&](const uint4& w, uint32_t* v) {
      if (a.wdt_bf16) {  // rounded as the weight conversion rounds
        float o[8];
        unpack8_bf16(w, o);
        v[0] = pack_half2(o[0], o[1]);
        v[1] = pack_half2(o[2], o[3]);
        v[2] = pack_half2(o[4], o[5]);
        v[3] = pack_half2(o[6], o[7]);
      } else {
        v[0] = w.x;
        v[1] = w.y;
        v[2] = w.z;
        v[3] = w.w;
      }
    };
    // the per-channel parameters of the current tile
    auto load_params = [&]() {
#pragma unroll
      for (int q = 0; q < kN / 2; ++q) {
        A2[q].x = cok ? -expf(a.A_log[c * kN + 2 * q]) * kLog2e : 0.0f;
        A2[q].y = cok ? -expf(a.A_log[c * kN + 2 * q + 1]) * kLog2e : 0.0f;
      }
      bias = cok ? a.dt_bias[c] : 0.f;
      Dc = cok ? a.D[c] : 0.f;
#pragma unroll
      for (int kx = 0; kx < kConv; ++kx) cw[kx] = cok ? bf(a.conv_w[c * kConv + kx]) : 0.f;
      cb = cok ? bf(a.conv_b[c]) : 0.f;
    };
    // the CTA's first tile: its W_dt rows from the ring, where the streamer put
    // them by TMA (zeros past R and past d), into TMEM
    auto load_first_tile = [&](int64_t tile) {
      cur_tile = tile;
      c = tile * kSC + cl;
      cok = c < a.d;
      const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
      mbar_wait(smem_u32(wfull), 0u, a.err, 48);
      for (int qs = 0; qs < a.nslab * 2; ++qs) {  // 16 columns = 32 K values of box qs / 2
        const uint8_t* rowp = stages + (qs >> 1) * (kSC * 128) + cl * 128;
        uint32_t v[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = (qs & 1) * 4 + e;  // 16-byte chunk of the row, stored at q ^ (row % 8)
          to_half8(*reinterpret_cast<const uint4*>(rowp + ((q ^ (cl & 7)) << 4)), v + 4 * e);
        }
        tmem_st16(trow + (uint32_t)(qs * 16), v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(wready));
        mbar_arrive(smem_u32(wcopied));
      }
      load_params();
    };
    // a later channel tile: its W_dt rows into TMEM (zeros past R and past d),
    // 16 loads in flight per thread at a time, then the per-channel parameters
    auto load_tile = [&](int64_t tile) {
      cur_tile = tile;
      c = tile * kSC + cl;
      cok = c < a.d;
      const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
      const int nq = a.nslab * 2;  // steps of 16 columns = 32 K values
      for (int q0 = 0; q0 < nq; q0 += 4) {
        uint4 w8[4][4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kx = (q0 + qq) * 32 + e * 8;
            w8[qq][e] = (cok && q0 + qq < nq && kx < a.R)
                            ? __ldg(reinterpret_cast<const uint4*>(a.wdt + c * a.R + kx))
                            : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          if (q0 + qq >= nq) break;
          uint32_t v[16];
#pragma unroll
          for (int e = 0; e < 4; ++e) to_half8(w8[qq][e], v + 4 * e);
          tmem_st16(trow + (uint32_t)((q0 + qq) * 16), v);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(wready));
      load_params();
    };
    // The first tile's W_dt (an input, or its copy prepared before the call) is
    // read before griddepcontrol.wait.
    if (g0 < g1) load_first_tile(g0 / ngrp);
    grid_dep_wait();  // dt_n and B/C come from the norms kernel
    // A row's new SSM and conv state go to global memory through the warp's
    // scratch rows (64-byte swizzled like the stage): one tensor store and one
    // bulk store issued by lane 0, whose reads of the scratch are waited for
    // only one row later, so the stores leave the row's dependency chain.
    uint8_t* wb = wb_s + warp * kDecWb;
    bool pend = false;
    auto wb_flush = [&]() {
      // the tensor store of one row ago has read the scratch (lane 0 issued it)
      if (!pend) return;
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      pend = false;
    };
    int64_t p = p0, i = 0;
    bool ok = true;
    for (int64_t g = g0, k = 0; ok && g < g1; ++g, ++k) {
      const int bsel = (int)(k & 1);
      const int64_t tile = g / ngrp, r0 = (g % ngrp) * kDB;
      if (tile != cur_tile) load_tile(tile);
      if (!mbar_wait(smem_u32(&mma_done[bsel]), (uint32_t)(k >> 1) & 1u, a.err, 45)) break;
      tc_fence_after();
      const uint32_t tacc =
          tmem + ((uint32_t)(warp * 32) << 16) + kDecAccCol + (uint32_t)(bsel * kDB);
      const float4* bcs = reinterpret_cast<const float4*>(bc_s + bsel * kDecBC);
      // the group's rows that fall in [p0, p1): pairs [lo, hi)
      const int64_t gp0 = tile * a.B + r0;  // pair of the group's first row
      const int64_t lo = p0 > gp0 ? p0 : gp0;
      const int64_t gend = gp0 + ((a.B - r0) < kDB ? (a.B - r0) : kDB);
      const int64_t hi = p1 < gend ? p1 : gend;
      // the group's 16 accumulators in one TMEM load; the rows are taken in
      // order, so the current row's value is kept in racc[0] by shifting
      uint32_t racc[kDB];
      tmem_ld16(tacc, racc);
      tmem_ld_wait();
      for (int q = (int)(lo - gp0); q > 0; --q) {
#pragma unroll
        for (int e = 0; e < kDB - 1; ++e) racc[e] = racc[e + 1];
      }
      for (p = lo; p < hi; ++p, ++i) {
        const int s = (int)(i % kDecStages);
        const int j = (int)(p - gp0);
        if (!mbar_wait(smem_u32(&full[s]), (uint32_t)(i / kDecStages) & 1u, a.err, 46)) {
          ok = false;
          break;
        }
        const int64_t b = r0 + j;
        const int64_t sl = dec_slot(a, b);
        // read the stage (state rows are 64-byte swizzled: 16-byte chunk q of
        // row cl sits at chunk q ^ ((cl >> 1) & 3)), then release it
        const uint8_t* st = stages + s * kDecStage;
        float2 h[kN / 2];
        float sv[kConv - 1];
        float xt, zv;
        const uint32_t xraw = reinterpret_cast<const uint16_t*>(st + kDecState + kDecConv)[cl];
        const uint32_t zraw =
            reinterpret_cast<const uint16_t*>(st + kDecState + kDecConv + kDecRow)[cl];
        xt = __uint_as_float(xraw << 16);
        zv = __uint_as_float(zraw << 16);
        if (sl >= 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(
                st + cl * 64 + 16 * (q ^ ((cl >> 1) & 3)));
            h[2 * q] = make_float2(v.x, v.y);
            h[2 * q + 1] = make_float2(v.z, v.w);
          }
          const uint16_t* cs = reinterpret_cast<const uint16_t*>(st + kDecState) + cl * 3;
#pragma unroll
          for (int kx = 0; kx < kConv - 1; ++kx) sv[kx] = __uint_as_float((uint32_t)cs[kx] << 16);
        } else {
#pragma unroll
          for (int q = 0; q < kN / 2; ++q) h[q] = make_float2(0.f, 0.f);
#pragma unroll
          for (int kx = 0; kx < kConv - 1; ++kx) sv[kx] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        if (sl < 0) {
          if (cl == 0 && atomicExch(&a.err->bad_input, 1u) == 0u) a.err->where = kSiteBadSlot;
#pragma unroll
          for (int e = 0; e < kDB - 1; ++e) racc[e] = racc[e + 1];  // the next row's first
          continue;
        }
        float xc = fmaf(cw[0], sv[0], cb);
        xc = fmaf(cw[1], sv[1], xc);
        xc = fmaf(cw[2], sv[2], xc);
        xc = fmaf(cw[3], xt, xc);
        const float uv = silu_u(xc);
        const float dl = softplus_fast(__uint_as_float(racc[0]) + bias);
#pragma unroll
        for (int e = 0; e < kDB - 1; ++e) racc[e] = racc[e + 1];  // the next row's first
        const float2 dl2 = make_float2(dl, dl), du2 = make_float2(dl * uv, dl * uv);
        float2 acc[4];
#pragma unroll
        for (int q4 = 0; q4 < kN / 4; ++q4) {
          const float4 Bq = bcs[j * 8 + q4];
          const float4 Cq = bcs[j * 8 + 4 + q4];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int q = q4 * 2 + half;
            const float2 Bp = half ? make_float2(Bq.z, Bq.w) : make_float2(Bq.x, Bq.y);
            const float2 Cp = half ? make_float2(Cq.z, Cq.w) : make_float2(Cq.x, Cq.y);
            const float2 xq = __fmul2_rn(dl2, A2[q]);
            const float2 da = make_float2(ex2_approx(xq.x), ex2_approx(xq.y));
            if constexpr (kZoh) {
              // 1 / A = 1 / (A2 ln 2); this path is not the hot one, so it divides
              const float2 inv_a = make_float2(kLog2e / A2[q].x, kLog2e / A2[q].y);
              h[q] = __ffma2_rn(da, h[q],
                                __fmul2_rn(__fmul2_rn(zoh_factor(xq, da, inv_a, dl2),
                                                      make_float2(uv, uv)),
                                           Bp));
            } else {
              h[q] = __ffma2_rn(da, h[q], __fmul2_rn(du2, Bp));
            }
            acc[q4] = half ? __ffma2_rn(Cp, h[q], acc[q4]) : __fmul2_rn(Cp, h[q]);
          }
        }
        if (cok) {  // (no divergent exit: the next row starts with a warp-wide TMEM load)
          const float2 sa = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
          const float ys = (sa.x + sa.y) + Dc * uv;
          a.y[b * a.d + c] = __float2bfloat16_rn(ys * silu_gate(zv));
        }
        // the previous row's stores have read the scratch; this row's state goes into it
        wb_flush();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4*>(wb + lane * 64 + 16 * (q ^ ((lane >> 1) & 3))) =
              make_float4(h[2 * q].x, h[2 * q].y, h[2 * q + 1].x, h[2 * q + 1].y);
        uint16_t* csw = reinterpret_cast<uint16_t*>(wb + 32 * 64) + lane * 3;
        csw[0] = (uint16_t)(__float_as_uint(sv[1]) >> 16);
        csw[1] = (uint16_t)(__float_as_uint(sv[2]) >> 16);
        csw[2] = (uint16_t)xraw;
        // one tensor store of the warp's [32 channels x 16] rows (channels past d
        // are outside the map and not written) and one bulk store of their conv
        // states, both reading the scratch
        const int64_t wc0 = c - lane;  // the warp's first channel
        const int64_t nv64 = a.d - wc0;
        const int nvalid = nv64 < 32 ? (int)nv64 : 32;  // of its channels that exist (may be <= 0)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && nvalid > 0) {
          tma_store_3d(&tm_state_wb, smem_u32(wb), 0, (int32_t)wc0, (int32_t)sl,
                       l2_evict_first_policy());
          bulk_store(a.conv_state + (sl * a.d + wc0) * (kConv - 1), smem_u32(wb + 32 * 64),
                     (uint32_t)(nvalid * 6));
          bulk_commit();
        }
        pend = true;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_free[bsel]));
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kDecTmemCols);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D tensor map of a row-major [rows, cols] matrix, box [box_rows, box_cols],
// with the given shared-memory swizzle.
bool make_map_swz(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base,
                  uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows,
                  CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tensor map of an SSM-state pool [slots, d, 16] fp32 with box [1, box_rows,
// 16] and 64-byte swizzle: a box never reaches past its slot's channels, so a
// tile store at the last channel tile writes only channels that exist.
bool make_state_map(CUtensorMap* m, const float* base, uint64_t slots, uint64_t d,
                    uint32_t box_rows = kSC) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kN, d, slots};
  cuuint64_t strides[2] = {(cuuint64_t)kN * 4, d * kN * 4};
  cuuint32_t box[3] = {(cuuint32_t)kN, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tensor map of x_proj's partial sums [S, T, P] fp32 with box [1, 32 rows,
// 16 columns] and the 64-byte swizzle: a box store never reaches past T or P.
bool make_part_map(CUtensorMap* m, const float* base, uint64_t S, uint64_t T, uint64_t P) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {P, T, S};
  cuuint64_t strides[2] = {P * 4, T * P * 4};
  cuuint32_t box[3] = {16, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tensor map of y [B, L, d] bf16 with box [1, 32 tokens, 128 channels]: a
// tile store never reaches past its sequence's tokens or past d.
bool make_y_map(CUtensorMap* m, const void* y, uint64_t B, uint64_t L, uint64_t d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d, L, B};
  cuuint64_t strides[2] = {d * 2, L * d * 2};
  cuuint32_t box[3] = {(cuuint32_t)kSC, (cuuint32_t)kSQ, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(y), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// As make_map_swz with the 128-byte swizzle (swz) or none.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base,
              uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows, bool swz) {
  return make_map_swz(m, dt, esize, base, rows, cols, box_cols, box_rows,
                      swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

struct FastWs {
  char* hdr;
  float* part;
  __half* u;
  __half* dtn;
  float* bc;
  __half* wx;
  __half* wdt;
  float4* ctab;       // k_xproj_conv: the conv weights and biases as its float32 table
  int* sched;         // [0] unit counter, [1..] hand-over flags of the scan's parts
  float* carry_h;     // scan hand-over: end state per (pair, part)
  float* carry_s;     // scan hand-over: sum of delta per (pair, part)
  int* order;         // packed batch: claim order of the sequences
  ScanPlan plan;
  size_t bytes;
  size_t zero_bytes;  // error header + scheduler words, cleared each call
  int ksplit;
};


// x_proj split over d_inner: about two CTAs per SM of a B200 (2 x 148), at
// most JMIX_XSPLIT_MAX splits, at least one 64-channel chunk per split.  Depends on the
// problem only, so the workspace size does too.
int xproj_ksplit(int64_t T, int64_t d) {
  if (T <= 0) return 1;
  const int64_t mtiles = (T + kXM - 1) / kXM;
  const int64_t kchunks = (d + kXK - 1) / kXK;
  int64_t ks = (JMIX_XPROJ_CTAS + 2 * mtiles - 1) / (2 * mtiles);  // 2 column parts
  if (ks > JMIX_XSPLIT_MAX) ks = JMIX_XSPLIT_MAX;
  if (ks > kchunks) ks = kchunks;
  return ks < 1 ? 1 : (int)ks;
}

#ifndef JMIX_XCONV
#define JMIX_XCONV 1  // prefill of sequences of one length: conv inside x_proj (k_xproj_conv)
#endif
// Whether steps 1-3 run as k_xproj_conv (plus k_norms16 when split): prefill
// (sequences of one length or a packed batch), dt_rank a multiple of 16; a
// decode step runs k_conv_step, k_xproj and k_norms16 (the conv spread over
// every SM: inside x_proj it measured slower at 256 rows).  Depends on the
// problem's shape only.
bool use_xconv(const Problem& pr) {
  return JMIX_XCONV && !pr.decode && pr.R % 16 == 0 && pr.T > 0;
}

// k_xproj_conv's split over d_inner: one split once the token tiles fill the
// GPU's 148 SMs (the norms then run in its epilogue), else enough splits for
// about one CTA per SM.
int xconv_ksplit(int64_t T, int64_t d) {
  const int64_t mtiles = (T + kXM - 1) / kXM;
  const int64_t kchunks = (d + kXK - 1) / kXK;
  if (mtiles >= 148) return 1;
  int64_t ks = (148 + mtiles - 1) / mtiles;
  if (ks > JMIX_XSPLIT_MAX) ks = JMIX_XSPLIT_MAX;
  if (ks > kchunks) ks = kchunks;
  return ks < 1 ? 1 : (int)ks;
}

FastWs fast_layout(const Problem& pr, char* base) {
  FastWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off = align256(off + n);
    return base ? base + o : nullptr;
  };
  const size_t T = (size_t)pr.T, d = (size_t)pr.d, P = (size_t)pr.P, R = (size_t)pr.R;
  const bool xconv = use_xconv(pr);
  w.ksplit = xconv ? xconv_ksplit(pr.T, pr.d) : xproj_ksplit(pr.T, pr.d);
  if (!pr.decode && !pr.cu) w.plan = scan_plan(pr.B, pr.L, pr.d);  // packed: one part each
  // hand-over slots: one per (pair, part) when parts exist
  const size_t slots = w.plan.n_parts > 1
                           ? (size_t)pr.B * (size_t)((pr.d + kSC - 1) / kSC) * w.plan.n_parts
                           : 0;
  w.hdr = take(sizeof(ErrFlags));
  w.sched = reinterpret_cast<int*>(take((1 + slots) * 4));
  w.zero_bytes = off;
  w.carry_h = reinterpret_cast<float*>(take(slots * kSC * kN * 4));
  w.carry_s = reinterpret_cast<float*>(take(slots * kSC * 4));
  w.order = pr.cu ? reinterpret_cast<int*>(take((size_t)pr.B * 4)) : nullptr;
  // (k_xproj_conv with one split writes no partial sums, and never u)
  w.part = reinterpret_cast<float*>(take(xconv && w.ksplit == 1 ? 0 : (size_t)w.ksplit * T * P * 4));
  w.u = reinterpret_cast<__half*>(take(xconv ? 0 : T * d * 2));
  w.dtn = reinterpret_cast<__half*>(take(T * R * 2));
  w.bc = reinterpret_cast<float*>(take(T * 2 * kN * 4));
  w.wx = reinterpret_cast<__half*>(take(P * d * 2));
  w.wdt = reinterpret_cast<__half*>(take(d * R * 2));
  w.ctab = reinterpret_cast<float4*>(take(xconv ? (d + kXK - 1) / kXK * kFTabBytes : 0));
  w.bytes = off;
  if (pr.prepared) {  // fp16 copies made once by jm_prepare_weights: W_x, then W_dt
    char* pw = static_cast<char*>(const_cast<void*>(pr.prepared));
    w.wx = reinterpret_cast<__half*>(pw);
    w.wdt = reinterpret_cast<__half*>(pw + align256(P * d * 2));
  }
  return w;
}

// Launch with programmatic stream serialisation: the kernel may start its
// prologue while the previous kernel on the stream finishes (once every CTA of
// that kernel has executed griddepcontrol.launch_dependents); it reads the
// previous kernels' results only after griddepcontrol.wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, unsigned block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// SM count of the current device, cached per device (threads that race on a
// slot store the same value).
int num_sms() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  int n = dev < kMaxDev ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    if (dev < kMaxDev) cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Whether a decode step's conv runs as k_conv_step (32-bit index arithmetic).
bool conv_step_fits(const Problem& p) {
  if (!p.decode) return false;
  const int64_t n_step = (p.d / 8) * ((p.B + kStepRows - 1) / kStepRows);
  const int64_t n_wx8 = p.prepared ? 0 : (int64_t)p.P * p.d / 8;
  return n_step + n_wx8 + 2048 < (int64_t)INT32_MAX && p.B < (int64_t)INT32_MAX &&
         p.n_slots < (int64_t)INT32_MAX && p.d < (int64_t)INT32_MAX;
}

cudaError_t run_fast_fwd(Problem& p) {
  FastWs w = fast_layout(p, p.ws);
  cudaStream_t s = p.stream;
  ErrFlags* err = reinterpret_cast<ErrFlags*>(w.hdr);
  // a prefill's weight preparation and a decode step's conv kernel clear the
  // error header and scheduler words themselves (so they can follow the kernel
  // before them with programmatic dependent launch); other calls clear them
  // with a memset first
  const bool xconv = use_xconv(p);
  const bool step_conv = !xconv && conv_step_fits(p);
  cudaError_t e = cudaSuccess;
  if (!xconv && !step_conv) {
    e = cudaMemsetAsync(p.ws, 0, w.zero_bytes, s);
    if (e != cudaSuccess) return e;
  }
  launches_begin(p);

  if (xconv) {
    // 1-3. W_x, W_dt -> fp16 (unless prepared once beforehand) and the conv
    // weight table; conv + SiLU inside x_proj; the norms in its epilogue (one
    // split) or after it
    {
      const int64_t n_wx8 = p.prepared ? 0 : (int64_t)p.P * p.d / 8;
      const int64_t n_wdt8 = p.prepared ? 0 : p.d * p.R / 8;
      const int64_t n_tab = (p.d + kXK - 1) / kXK * kFTabUnits;
      e = launch_pdl(k_convert_weights, dim3((unsigned)((n_wx8 + n_wdt8 + n_tab + 255) / 256)),
                     256, 0, s, (const bf16*)p.xproj_w, n_wx8, w.wx, (const bf16*)p.dtproj_w,
                     n_wdt8, w.wdt, (const bf16*)p.conv_w, (const bf16*)p.conv_b, p.d, w.ctab,
                     n_tab, reinterpret_cast<unsigned*>(p.ws), (int)(w.zero_bytes / 4));
      if (e != cudaSuccess) return e;
      launched(p, "k_convert_weights");
    }
    CUtensorMap tx, tw;
    XconvArgs xa;
    xa.T = p.T;
    xa.L = p.L;
    xa.d = p.d;
    xa.P = (int)p.P;
    xa.R = (int)p.R;
    xa.N1 = (int)(((p.P + 1) / 2 + 15) / 16 * 16);  // two MMAs of N1 columns
    xa.kchunks = (int)((p.d + kXK - 1) / kXK);
    xa.ksplit = w.ksplit;
    xa.tmem_cols = 2 * xa.N1 <= 64 ? 64 : 2 * xa.N1 <= 128 ? 128 : 2 * xa.N1 <= 256 ? 256 : 512;
    xa.ctab = w.ctab;
    xa.hist = (const bf16*)p.init_conv;
    xa.cu = p.cu;
    xa.nseq = p.B;
    xa.part = w.part;
    xa.dtn_w = (const bf16*)p.dtn_w;
    xa.bn_w = (const bf16*)p.bn_w;
    xa.cn_w = (const bf16*)p.cn_w;
    xa.eps = p.eps;
    xa.dtn = w.dtn;
    xa.bc = w.bc;
    xa.err = err;
    if (!make_map_swz(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x, p.T, p.d, kXK, kFXRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.wx, p.P, p.d, kXK, xa.N1, true))
      return cudaErrorInvalidValue;
    CUtensorMap tp;  // the partial sums [ksplit, T, P] (several splits), boxes of 16 x 32
    if (xa.ksplit > 1 && !make_part_map(&tp, w.part, (uint64_t)xa.ksplit, (uint64_t)p.T,
                                        (uint64_t)p.P))
      return cudaErrorInvalidValue;
    if (xa.ksplit == 1) tp = tw;  // (not read with one split)
    cudaFuncSetAttribute(k_xproj_conv, cudaFuncAttributeMaxDynamicSharedMemorySize, kFSmem);
    const dim3 grid((unsigned)((p.T + kXM - 1) / kXM), (unsigned)xa.ksplit);
    e = launch_pdl(k_xproj_conv, grid, kFThreads, (size_t)kFSmem, s, tx, tw, tp, xa);
    if (e != cudaSuccess) return e;
    launched(p, "k_xproj_conv");
    if (w.ksplit > 1) {
      if (w.ksplit <= 4)
        e = launch_pdl(k_norms16_warp<bf16>, dim3((unsigned)((p.T + 7) / 8)), 256, 0, s, w.part,
                       w.ksplit, (const bf16*)p.dtn_w, (const bf16*)p.bn_w,
                       (const bf16*)p.cn_w, p.T, (int)p.R, p.eps, w.dtn, w.bc);
      else
        e = launch_pdl(k_norms16<bf16, 1>, dim3((unsigned)p.T), kNormThreads, 0, s, w.part,
                       w.ksplit, (const bf16*)p.dtn_w, (const bf16*)p.bn_w,
                       (const bf16*)p.cn_w, p.T, (int)p.R, p.eps, w.dtn, w.bc);
      if (e != cudaSuccess) return e;
      launched(p, "k_norms16");
    }
  } else {
    // 1. conv + SiLU -> u (fp16); weights -> fp16 (unless prepared once beforehand)
    {
      const int G = p.L >= kConvG ? kConvG : 1;
      const int64_t n_conv = (p.d / 8) * ((p.L + G - 1) / G) * p.B;
      const int64_t n_wx8 = p.prepared ? 0 : (int64_t)p.P * p.d / 8;
      // (a decode step rounds W_dt to fp16 as it loads it into TMEM)
      const int64_t n_wdt8 = (p.prepared || p.decode) ? 0 : p.d * p.R / 8;
      const int64_t total = n_conv + n_wx8 + n_wdt8;
      const int64_t n_step = (p.d / 8) * ((p.B + kStepRows - 1) / kStepRows);
      const int64_t n_cvt = (n_wx8 + kStepCvt - 1) / kStepCvt;
      const bool step = step_conv;
      if (step) {
        e = launch_pdl(k_conv_step, dim3((unsigned)((n_step + n_cvt + 255) / 256)), 256, 0, s,
                       (const bf16*)p.x, (const bf16*)p.conv_w, (const bf16*)p.conv_b,
                       (const bf16*)p.init_conv, p.sidx, (int)p.n_slots, (int)p.B, (int)p.d, w.u,
                       (int)n_step, (const bf16*)p.xproj_w, (int)n_wx8, w.wx,
                       reinterpret_cast<unsigned*>(p.ws), (int)(w.zero_bytes / 4));
        if (e != cudaSuccess) return e;
      } else if (p.cu) {
        const int64_t n_pk = (p.d / 8) * ((p.T + 7) / 8);
        k_conv_silu16_packed<<<(unsigned)((n_pk + n_wx8 + n_wdt8 + 255) / 256), 256, 0, s>>>(
            (const bf16*)p.x, (const bf16*)p.conv_w, (const bf16*)p.conv_b,
            (const bf16*)p.init_conv, p.cu, p.B, p.T, p.d, w.u, n_pk, (const bf16*)p.xproj_w,
            n_wx8, w.wx, (const bf16*)p.dtproj_w, n_wdt8, w.wdt);
      } else {
        auto kern = G == kConvG ? k_conv_silu16<kConvG> : k_conv_silu16<1>;
        kern<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
            (const bf16*)p.x, (const bf16*)p.conv_w, (const bf16*)p.conv_b,
            (const bf16*)p.init_conv, p.sidx, p.n_slots, p.B, p.L, p.d, w.u, n_conv,
            (const bf16*)p.xproj_w, n_wx8, w.wx, (const bf16*)p.dtproj_w, n_wdt8, w.wdt);
      }
      launched(p, step ? "k_conv_step" : "k_conv_silu16");
    }
    // 2. x_proj on tcgen05
    {
      CUtensorMap tu, tw;
      XprojArgs xa;
      xa.T = p.T;
      xa.P = (int)p.P;
      // two column parts of N1 (a multiple of 16), one per CTA of the grid's z
      xa.N1 = (int)(((p.P + 1) / 2 + 15) / 16 * 16);
      xa.N2 = xa.N1;
      xa.Ntot = xa.N1 + xa.N2;
      xa.kchunks = (int)((p.d + kXK - 1) / kXK);
      const int64_t mtiles = (p.T + kXM - 1) / kXM;
      xa.ksplit = w.ksplit;
      xa.tmem_cols = xa.N1 <= 32 ? 32 : xa.N1 <= 64 ? 64 : xa.N1 <= 128 ? 128 : 256;
      xa.part = w.part;
      xa.err = err;
      if (!make_map(&tu, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.u, p.T, p.d, kXK, kXM, true) ||
          !make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.wx, p.P, p.d, kXK, xa.N1, true))
        return cudaErrorInvalidValue;
      CUtensorMap tp;  // the partial sums [ksplit, T, P], boxes of 16 columns x 32 rows
      if (!make_part_map(&tp, w.part, (uint64_t)xa.ksplit, (uint64_t)p.T, (uint64_t)p.P))
        return cudaErrorInvalidValue;
      const int smem = 1024 + kXStages * (kXM * 128 + xa.N1 * 128) + 256;
      cudaFuncSetAttribute(k_xproj, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      e = launch_pdl(k_xproj, dim3((unsigned)(2 * mtiles), (unsigned)xa.ksplit), kXThreads,
                     (size_t)smem, s, tu, tw, tp, xa);
      if (e != cudaSuccess) return e;
      launched(p, "k_xproj");
    }
    // 3. RMSNorms
    if (w.ksplit <= 4)
      e = launch_pdl(k_norms16_warp<bf16>, dim3((unsigned)((p.T + 7) / 8)), 256, 0, s, w.part,
                     w.ksplit, (const bf16*)p.dtn_w, (const bf16*)p.bn_w, (const bf16*)p.cn_w, p.T,
                     (int)p.R, p.eps, w.dtn, w.bc);
    else
      e = launch_pdl(k_norms16<bf16, 1>, dim3((unsigned)p.T), kNormThreads, 0, s, w.part, w.ksplit,
                     (const bf16*)p.dtn_w, (const bf16*)p.bn_w, (const bf16*)p.cn_w, p.T, (int)p.R,
                     p.eps, w.dtn, w.bc);
    if (e != cudaSuccess) return e;
    launched(p, "k_norms16");
  }
  // 4. dt_proj + scan + gate
  if (p.decode) {
    CUtensorMap tstate, tstate_wb, tdtn, tbc, twdt;
    const int64_t slots = p.sidx ? p.n_slots : p.B;
    if (!make_state_map(&tstate, p.final_state, (uint64_t)slots, (uint64_t)p.d) ||
        !make_state_map(&tstate_wb, p.final_state, (uint64_t)slots, (uint64_t)p.d, 32) ||
        !make_map(&tdtn, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.dtn, p.T, p.R, 64, kDB, true) ||
        !make_map(&tbc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, w.bc, p.T, 2 * kN, 2 * kN, kDB,
                  false))
      return cudaErrorInvalidValue;
    DecArgs da;
    da.B = p.B;
    da.d = p.d;
    da.R = (int)p.R;
    da.nslab = (int)((p.R + 63) / 64);
    da.n_tiles = (int)((p.d + kSC - 1) / kSC);
    da.pairs = p.B * da.n_tiles;
    da.x = (const bf16*)p.x;
    da.z = (const bf16*)p.z;
    da.conv_w = (const bf16*)p.conv_w;
    da.conv_b = (const bf16*)p.conv_b;
    da.dt_bias = p.dt_bias;
    da.A_log = p.A_log;
    da.D = p.D;
    // the prepared fp16 W_dt when there is one, else the bf16 input
    da.wdt = p.prepared ? reinterpret_cast<const uint16_t*>(w.wdt)
                        : reinterpret_cast<const uint16_t*>(p.dtproj_w);
    da.wdt_bf16 = p.prepared ? 0 : 1;
    // W_dt [d, R] in boxes of 64 K values x 128 channels (a CTA's first tile)
    if (!make_map(&twdt,
                  p.prepared ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  da.wdt, p.d, p.R, 64, kSC, true))
      return cudaErrorInvalidValue;
    da.conv_state = (bf16*)p.final_conv;
    da.ssm_state = p.final_state;
    da.y = (bf16*)p.y;
    da.err = err;
    da.sidx = p.sidx;
    da.n_slots = slots;
    auto dec_kern = p.zoh ? k_decode_scan<true> : k_decode_scan<false>;
    cudaFuncSetAttribute(dec_kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    const int64_t ctas = std::min<int64_t>(2 * num_sms(), da.pairs);
    e = launch_pdl(dec_kern, (unsigned)ctas, kDecThreads, kDecSmem, s, tstate, tstate_wb, tdtn,
                   tbc, twdt, da);
    if (e != cudaSuccess) return e;
    launched(p, "k_decode_scan");
  } else {
    CUtensorMap twdt, tdtn, tbc, tx, tz;
    if (!make_map(&twdt, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.wdt, p.d, p.R, 64, kSC, true) ||
        !make_map(&tdtn, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.dtn, p.T, p.R, 64, kSQ, true) ||
        !make_map(&tbc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, w.bc, p.T, 2 * kN, 2 * kN, kSQ,
                  false) ||
        !make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.x, p.T, p.d, kSC, kSQ, false) ||
        !make_map(&tz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.z, p.T, p.d, kSC, kSQ, false))
      return cudaErrorInvalidValue;
    ScanArgs sa;
    sa.L = p.L;
    sa.B = p.B;
    sa.cu = p.cu;
    sa.order = nullptr;
    if (p.cu && p.B > 1 && p.B <= 8192) {  // O(B^2) ranking: up to a few thousand prompts
      k_order_by_length<<<1, 1024, 0, s>>>(p.cu, (int)p.B, (int)p.T, w.order);
      launched(p, "k_order_by_length");
      sa.order = w.order;
    }
    sa.d = p.d;
    sa.T = p.T;
    sa.R = (int)p.R;
    sa.nslab = (int)((p.R + 63) / 64);
    sa.x = (const bf16*)p.x;
    sa.z = (const bf16*)p.z;
    sa.conv_w = (const bf16*)p.conv_w;
    sa.conv_b = (const bf16*)p.conv_b;
    sa.dt_bias = p.dt_bias;
    sa.A_log = p.A_log;
    sa.D = p.D;
    sa.h0 = p.init_ssm;
    sa.hT = p.final_state;
    sa.y = (bf16*)p.y;
    sa.hist = (const bf16*)p.init_conv;
    sa.final_conv = (bf16*)p.final_conv;
    sa.wdt = w.wdt;
    sa.err = err;
    sa.n_tiles = (int)((p.d + kSC - 1) / kSC);
    sa.n_parts = w.plan.n_parts;
    sa.two_pass = w.plan.two_pass;
    sa.counter = w.sched;
    sa.flags = w.sched + 1;
    sa.carry_h = w.carry_h;
    sa.carry_s = w.carry_s;
    const int pairs = sa.n_tiles * (int)p.B;
    const int units = pairs * sa.n_parts + (sa.two_pass ? pairs * (sa.n_parts - 1) : 0);
    const int slots = kScanCtasPerSm * num_sms();
    auto scan_kern = p.zoh ? k_scan_fused<true, JMIX_SCAN_LEAD != 0>
                           : k_scan_fused<false, JMIX_SCAN_LEAD != 0>;
    cudaFuncSetAttribute(scan_kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kScanSmem);
    cudaFuncSetAttribute(scan_kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    CUtensorMap ty;  // y as [B, L, d] (a packed batch stores y thread by thread)
    if (!make_y_map(&ty, p.y, p.cu ? 1 : (uint64_t)p.B, p.cu ? (uint64_t)p.T : (uint64_t)p.L,
                    (uint64_t)p.d))
      return cudaErrorInvalidValue;
    e = launch_pdl(scan_kern, dim3((unsigned)(units < slots ? units : slots)),
                   JMIX_SCAN_LEAD ? 128u : (unsigned)kScanThreads, (size_t)kScanSmem, s, twdt,
                   tdtn, tbc, tx, tz, ty, sa);
    if (e != cudaSuccess) return e;
    launched(p, "k_scan_fused");
  }
  return cudaGetLastError();
}

}  // namespace

size_t fast_ws_bytes(const Problem& p) { return fast_layout(p, nullptr).bytes; }

size_t prepared_weights_bytes(int64_t d, int64_t R) {
  return align256((size_t)(R + 2 * kN) * d * 2) + align256((size_t)d * R * 2);
}

// The fp16 copies of W_x and W_dt, rounded as a call's weight preparation
// rounds them (k_convert_weights with no conv table and no header to clear).
cudaError_t run_prepare_weights(int64_t d, int64_t R, const void* xproj_w, const void* dtproj_w,
                                void* out, cudaStream_t s) {
  const int64_t P = R + 2 * kN;
  const int64_t n_wx8 = P * d / 8, n_wdt8 = d * R / 8;
  __half* wx16 = static_cast<__half*>(out);
  __half* wdt16 = reinterpret_cast<__half*>(static_cast<char*>(out) + align256((size_t)P * d * 2));
  k_convert_weights<<<(unsigned)((n_wx8 + n_wdt8 + 255) / 256), 256, 0, s>>>(
      (const bf16*)xproj_w, n_wx8, wx16, (const bf16*)dtproj_w, n_wdt8, wdt16, nullptr, nullptr,
      d, nullptr, 0, nullptr, 0);
  return cudaGetLastError();
}

void fast_scan_schedule(int64_t B, int64_t L, int64_t d, int* n_parts, int* two_pass) {
  const ScanPlan pl = scan_plan(B, L, d);
  *n_parts = pl.n_parts;
  *two_pass = pl.two_pass;
}

cudaError_t run_fast(Problem& p) { return run_fast_fwd(p); }

}  // namespace jmix
