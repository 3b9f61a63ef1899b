// Backward of the selective-scan core (training), float32.
//
// Forward (Euler B; Jamba guide, "Inside the Mamba State-Space Layers"):
//   h_t = a_t h_{t-1} + delta_t B_t u_t,  a_t = exp(delta_t A),  A = -exp(A_log),
//   y_t = C_t . h_t + D u_t.
// Given gy = dLoss/dy, reverse mode gives, with g the gradient flowing into h_t:
//   g   += C_t gy_t;  gC_t += gy_t h_t;  gu_t = D gy_t + sum_n g_n delta_t B_t,n;
//   gB_t += g delta_t u_t;  gdelta_t = sum_n g_n (A_n a_t,n h_{t-1},n + B_t,n u_t);
//   gA_n += g_n delta_t a_t,n h_{t-1},n;  gD += gy_t u_t;  g <- a_t g  (to h_{t-1});
// and g_h0 = g after the first token, gA_log = gA * A.
//
// Time parts.  Each sequence is cut into P parts of whole chunks that run side by
// side.  Both recurrences are linear with the same decays, so a part acts on
// what enters it through one factor, exp(A S), S = sum of delta over the part:
//   forward:  h_end = exp(A S) h_start + f_p   (f_p: the part's end state from 0)
//   adjoint:  g_out = exp(A S) g_in + r_p      (r_p: the gradient the part sends
//             to h before it when nothing enters from its right; g_in is what
//             the part after it sends)
// k_scan_bwd_parts computes f_p, r_p and S for every part; each part of
// k_scan_bwd then folds them (forward over the parts before it, from h0;
// adjoint over the parts after it, from zero) into its own h_start and g_in.
//
// k_scan_bwd: CTA = (128-channel tile, sequence, part), thread = channel, 16
// states in registers.  Pass 1 runs the recurrence forward over the part and
// stores the state at the start of every kCk-token chunk.  Pass 2 walks the
// part's chunks backwards: it recomputes the chunk's states into shared memory
// ([token][state][channel], conflict-free) and runs the reverse recurrence
// token by token.  gB and gC are sums over channels: each warp reduces its 32
// channels' 32 values (16 gB, 16 gC) by a reduce-scatter of shuffles (lane i
// ends with index i) into a per-warp partial row; k_scan_bwd_reduce adds the
// partials in a fixed order, and gA_log, gD over the (sequence, part) rows, so
// the results are reproducible.
#include "jmix_internal.cuh"

#define JM_API extern "C" __attribute__((visibility("default")))

namespace jmix {
namespace {

constexpr int kBwdThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// exp(y) as MUFU ex2 of y log2(e), with y = delta A already scaled: the argument
// is A2 delta, A2 = A log2(e) (relative error ~2 ulp of ex2 plus the rounding of
// the product; far inside the 1e-4 gradient tolerance).
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr int kCk = 4;  // tokens per checkpoint chunk (32 KB of states in shared memory)
constexpr int kBwdMaxParts = 16;
constexpr int kPg = 8;  // tokens per load group in k_scan_bwd_parts
constexpr int kBwdMinPartChunks = 2;
// Resident k_scan_bwd CTAs on a B200: 3 per SM (154 registers x 128 threads).
constexpr int kBwdSlots = 3 * 148;

// Time parts per sequence.  Parts cost an extra kernel (two passes over the
// tokens), so a batch that already fills the GPU's CTA slots well runs as one
// part; otherwise P (at most kBwdMaxParts, parts of at least kBwdMinPartChunks
// chunks) maximises the filled fraction of the waves of (tile, sequence, part)
// CTAs, less 1% per part for the folds.
int bwd_parts(int64_t B, int64_t L, int64_t d) {
  const int64_t n_tiles = (d + kBwdThreads - 1) / kBwdThreads;
  const int64_t nck = (L + kCk - 1) / kCk;
  if (B <= 0 || nck <= 0) return 1;
  auto fill = [&](int64_t P) {
    const int64_t ctas = n_tiles * B * P;
    return (double)ctas / (double)(((ctas + kBwdSlots - 1) / kBwdSlots) * kBwdSlots);
  };
  if (fill(1) >= 0.9) return 1;
  int best = 1;
  double best_score = fill(1);
  for (int P = 2; P <= kBwdMaxParts && P * kBwdMinPartChunks <= nck; ++P) {
    const double score = fill(P) - 0.01 * (P - 1);
    if (score > best_score) {
      best_score = score;
      best = P;
    }
  }
  return best;
}

struct BwdArgs {
  int64_t B, L, d;
  const float* delta;
  const float* u;
  const float* Bm;
  const float* Cm;
  const float* A_log;
  const float* D;
  const float* h0;
  const float* gy;
  float* gdelta;
  float* gu;
  float* gh0;
  float* ckpt;      // [B, nck, d, 16]
  float* part_bc;   // [n_tiles * 4, B * L, 32]: per-warp sums of gB (0..15), gC (16..31)
  float* part_a;    // [P * B, d, 16]
  float* part_d;    // [P * B, d]
  int P;            // time parts per sequence
  float* f_end;     // [P * B, d, 16]: a part's end state from a zero start
  float* r_out;     // [P * B, d, 16]: a part's outgoing gradient with nothing entering
  float* s_sum;     // [P * B, d]: a part's sum of delta
};

// Chunks [k0, k1) of the sequence form part p.
__device__ __forceinline__ void part_chunks(int64_t nck, int P, int p, int64_t& k0, int64_t& k1) {
  k0 = nck * p / P;
  k1 = nck * (p + 1) / P;
}

// For each part: f_p (forward from a zero state), S (sum of delta) and r_p (the
// adjoint run backwards from a zero incoming gradient: g += C_t gy_t, g <- a_t g).
__global__ void __launch_bounds__(kBwdThreads) k_scan_bwd_parts(const BwdArgs a) {
  const int64_t b = blockIdx.y;
  const int p = blockIdx.z;
  const int64_t c = (int64_t)blockIdx.x * kBwdThreads + threadIdx.x;
  // a group's kPg rows of B (forward) or C (adjoint): kPg * 16 = 128 floats, one
  // per thread, double-buffered (one barrier per group)
  __shared__ float rows[2][kPg * kN];
  static_assert(kPg * kN == kBwdThreads, "one row element per thread");
  const bool cok = c < a.d;
  const int64_t L = a.L, d = a.d;
  const int64_t nck = (L + kCk - 1) / kCk;
  int64_t k0, k1;
  part_chunks(nck, a.P, p, k0, k1);
  const int64_t t0 = k0 * kCk, t1 = k1 * kCk < L ? k1 * kCk : L;
  const int ri = threadIdx.x / kN, rn = threadIdx.x % kN;  // this thread's row element
  float A2[kN];  // A log2(e)
#pragma unroll
  for (int n = 0; n < kN; ++n) A2[n] = cok ? -expf(a.A_log[c * kN + n]) * kLog2e : 0.0f;
  float h[kN], g[kN];
#pragma unroll
  for (int n = 0; n < kN; ++n) h[n] = g[n] = 0.0f;
  float S = 0.0f;
  // groups of kPg tokens: the group's per-channel loads go out before its
  // arithmetic, so their latency is paid once per group, not once per token
  int buf = 0;
  for (int64_t tg = t0; tg < t1; tg += kPg, buf ^= 1) {
    float dl[kPg], uv[kPg];
#pragma unroll
    for (int i = 0; i < kPg; ++i) {
      const int64_t t = tg + i < t1 ? tg + i : t1 - 1;
      dl[i] = cok ? a.delta[(b * L + t) * d + c] : 0.0f;
      uv[i] = cok ? a.u[(b * L + t) * d + c] : 0.0f;
    }
    rows[buf][threadIdx.x] = tg + ri < t1 ? a.Bm[(b * L + tg + ri) * kN + rn] : 0.0f;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kPg; ++i) {
      if (tg + i >= t1) break;
      const float du = dl[i] * uv[i];
      const float* Bt = rows[buf] + i * kN;
      S += dl[i];
#pragma unroll
      for (int n = 0; n < kN; ++n) h[n] = fmaf(ex2f(dl[i] * A2[n]), h[n], du * Bt[n]);
    }
  }
  for (int64_t tg = t1 - 1; tg >= t0; tg -= kPg, buf ^= 1) {  // tokens tg, tg-1, .. (>= t0)
    float dl[kPg], gyt[kPg];
#pragma unroll
    for (int i = 0; i < kPg; ++i) {
      const int64_t t = tg - i >= t0 ? tg - i : t0;
      dl[i] = cok ? a.delta[(b * L + t) * d + c] : 0.0f;
      gyt[i] = cok ? a.gy[(b * L + t) * d + c] : 0.0f;
    }
    rows[buf][threadIdx.x] = tg - ri >= t0 ? a.Cm[(b * L + tg - ri) * kN + rn] : 0.0f;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kPg; ++i) {
      if (tg - i < t0) break;
      const float* Ct = rows[buf] + i * kN;
#pragma unroll
      for (int n = 0; n < kN; ++n) g[n] = ex2f(dl[i] * A2[n]) * fmaf(Ct[n], gyt[i], g[n]);
    }
  }
  if (!cok) return;
  const int64_t row = ((int64_t)p * a.B + b) * d + c;
#pragma unroll
  for (int n = 0; n < kN; ++n) {
    a.f_end[row * kN + n] = h[n];
    a.r_out[row * kN + n] = g[n];
  }
  a.s_sum[row] = S;
}

// Sums v over the 32 lanes of the warp, index by index: afterwards lane i holds
// in v[0] the sum of every lane's v[i].
__device__ __forceinline__ void warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool up = lane & off;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = up ? v[i] : v[i + off];
      const float keep = up ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
}

__global__ void __launch_bounds__(kBwdThreads, 3) k_scan_bwd(const BwdArgs a) {
  __shared__ float hs[kCk][kN][kBwdThreads];  // states after each token of the chunk
  // the chunk's rows of B (0..15) and C (16..31): kCk * 32 = 128 floats, one per
  // thread, double-buffered (one barrier per chunk)
  __shared__ float bcrow[2][kCk * 2 * kN];
  static_assert(kCk * 2 * kN == kBwdThreads, "one row element per thread");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b = blockIdx.y;
  const int p = blockIdx.z, P = a.P;
  const int64_t c = (int64_t)blockIdx.x * kBwdThreads + threadIdx.x;
  const bool cok = c < a.d;
  const int64_t L = a.L, d = a.d;
  const int64_t nck = (L + kCk - 1) / kCk;
  int64_t k0, k1;
  part_chunks(nck, P, p, k0, k1);
  float A2[kN];  // A log2(e)
#pragma unroll
  for (int n = 0; n < kN; ++n) A2[n] = cok ? -expf(a.A_log[c * kN + n]) * kLog2e : 0.0f;
  const float Dc = cok ? a.D[c] : 0.0f;
  auto at = [&](const float* q, int64_t t) { return cok ? q[(b * L + t) * d + c] : 0.0f; };
  // this thread's element of chunk j's B/C rows
  const int ri = threadIdx.x / (2 * kN), rk = threadIdx.x % (2 * kN);
  auto stage_rows = [&](int64_t j, int buf) {
    const int64_t t = j * kCk + ri;
    bcrow[buf][threadIdx.x] =
        t < L ? (rk < kN ? a.Bm[(b * L + t) * kN + rk] : a.Cm[(b * L + t) * kN + rk - kN]) : 0.0f;
    __syncthreads();
  };
  int buf = 0;
  // the part's start state: h0 folded through the parts before it
  float h[kN];
#pragma unroll
  for (int n = 0; n < kN; ++n) h[n] = (cok && a.h0) ? a.h0[(b * d + c) * kN + n] : 0.0f;
  for (int q = 0; q < p && cok; ++q) {
    const int64_t row = ((int64_t)q * a.B + b) * d + c;
    const float S = a.s_sum[row];
#pragma unroll
    for (int n = 0; n < kN; ++n) h[n] = fmaf(ex2f(A2[n] * S), h[n], a.f_end[row * kN + n]);
  }
  // pass 1: forward, checkpoint at every chunk start; a chunk's loads go out
  // before its arithmetic
  for (int64_t j = k0; j < k1; ++j) {
    const int64_t t0 = j * kCk;
    const int nt = (int)((L - t0) < kCk ? (L - t0) : kCk);
    if (cok) {
      float* ck = a.ckpt + ((b * nck + j) * d + c) * kN;
#pragma unroll
      for (int n = 0; n < kN; ++n) ck[n] = h[n];
    }
    float dl[kCk], uv[kCk];
#pragma unroll
    for (int i = 0; i < kCk; ++i) {
      dl[i] = i < nt ? at(a.delta, t0 + i) : 0.0f;
      uv[i] = i < nt ? at(a.u, t0 + i) : 0.0f;
    }
    stage_rows(j, buf);
#pragma unroll
    for (int i = 0; i < kCk; ++i) {
      if (i >= nt) break;
      const float du = dl[i] * uv[i];
      const float* Bt = bcrow[buf] + i * 2 * kN;
#pragma unroll
      for (int n = 0; n < kN; ++n) h[n] = fmaf(ex2f(dl[i] * A2[n]), h[n], du * Bt[n]);
    }
    buf ^= 1;
  }
  // pass 2: reverse, from the gradient the parts after this one send into it
  float g[kN], gA[kN], gD = 0.0f;
#pragma unroll
  for (int n = 0; n < kN; ++n) g[n] = gA[n] = 0.0f;
  for (int q = P - 1; q > p && cok; --q) {
    const int64_t row = ((int64_t)q * a.B + b) * d + c;
    const float S = a.s_sum[row];
#pragma unroll
    for (int n = 0; n < kN; ++n) g[n] = fmaf(ex2f(A2[n] * S), g[n], a.r_out[row * kN + n]);
  }
  const int64_t tile_warp = (int64_t)blockIdx.x * 4 + warp;
  for (int64_t j = k1 - 1; j >= k0; --j) {
    const int64_t t0 = j * kCk;
    const int nt = (int)((L - t0) < kCk ? (L - t0) : kCk);
    float hstart[kN];
    if (cok) {
      const float* ck = a.ckpt + ((b * nck + j) * d + c) * kN;
#pragma unroll
      for (int n = 0; n < kN; ++n) hstart[n] = ck[n];
    } else {
#pragma unroll
      for (int n = 0; n < kN; ++n) hstart[n] = 0.0f;
    }
    float dlc[kCk], uvc[kCk], gyc[kCk];  // the chunk's per-channel inputs
#pragma unroll
    for (int i = 0; i < kCk; ++i) {
      dlc[i] = i < nt ? at(a.delta, t0 + i) : 0.0f;
      uvc[i] = i < nt ? at(a.u, t0 + i) : 0.0f;
      gyc[i] = i < nt ? at(a.gy, t0 + i) : 0.0f;
    }
    stage_rows(j, buf);
#pragma unroll
    for (int n = 0; n < kN; ++n) h[n] = hstart[n];
#pragma unroll
    for (int i = 0; i < kCk; ++i) {
      if (i >= nt) break;
      const float du = dlc[i] * uvc[i];
      const float* Bt = bcrow[buf] + i * 2 * kN;
#pragma unroll
      for (int n = 0; n < kN; ++n) {
        h[n] = fmaf(ex2f(dlc[i] * A2[n]), h[n], du * Bt[n]);
        hs[i][n][threadIdx.x] = h[n];
      }
    }
#pragma unroll
    for (int i = kCk - 1; i >= 0; --i) {
      if (i >= nt) continue;
      const int64_t t = t0 + i;
      const float dl = dlc[i], uv = uvc[i], gyt = gyc[i];
      const float* Bt = bcrow[buf] + i * 2 * kN;
      const float* Ct = Bt + kN;
      float v[32];  // this channel's share of gB_t (0..15) and gC_t (16..31)
      // gdelta = sum_n g_n (A_n a_n h_{t-1},n + B_n u) = ln2 s_a + u s_b and
      // gu = D gy + delta s_b, with s_a = sum_n g_n A2_n a_n h_{t-1},n, s_b = sum_n g_n B_n
      float s_a = 0.0f, s_b = 0.0f;
      gD = fmaf(gyt, uv, gD);
#pragma unroll
      for (int n = 0; n < kN; ++n) {
        const float an = ex2f(dl * A2[n]);
        const float hp = i > 0 ? hs[i - 1][n][threadIdx.x] : hstart[n];
        const float ht = hs[i][n][threadIdx.x];
        g[n] = fmaf(Ct[n], gyt, g[n]);
        v[16 + n] = gyt * ht;
        s_b = fmaf(g[n], Bt[n], s_b);
        v[n] = g[n] * dl * uv;
        s_a = fmaf(g[n] * A2[n] * an, hp, s_a);
        gA[n] = fmaf(g[n] * dl * an, hp, gA[n]);
        g[n] *= an;
      }
      const float gdl = fmaf(kLn2, s_a, uv * s_b);
      const float gut = fmaf(dl, s_b, Dc * gyt);
      if (!cok) {
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = 0.0f;
      }
      if (cok) {
        a.gdelta[(b * L + t) * d + c] = gdl;
        a.gu[(b * L + t) * d + c] = gut;
      }
      warp_reduce_scatter32(v, lane);
      a.part_bc[(tile_warp * (a.B * L) + b * L + t) * 32 + lane] = v[0];
    }
    buf ^= 1;
  }
  if (cok) {
    const int64_t row = ((int64_t)p * a.B + b) * d + c;
#pragma unroll
    for (int n = 0; n < kN; ++n) a.part_a[row * kN + n] = gA[n];
    a.part_d[row] = gD;
    if (a.gh0 && p == 0)
#pragma unroll
      for (int n = 0; n < kN; ++n) a.gh0[(b * d + c) * kN + n] = g[n];
  }
}

// gB, gC: sum over the per-warp partial rows, in order; gA_log, gD: sum over
// the (part, sequence) rows, in order, then gA_log = gA * A.
__global__ void k_scan_bwd_reduce(const float* __restrict__ part_bc, int64_t n_rows, int64_t TB,
                                  const float* __restrict__ part_a, const float* __restrict__ part_d,
                                  const float* __restrict__ A_log, int64_t n_ad, int64_t d,
                                  float* __restrict__ gB, float* __restrict__ gC,
                                  float* __restrict__ gA_log, float* __restrict__ gD) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n_bc = TB * 32;
  if (i < n_bc) {
    float s = 0.0f;
    for (int64_t r = 0; r < n_rows; ++r) s += part_bc[r * n_bc + i];
    const int64_t tok = i >> 5;
    const int k = (int)(i & 31);
    if (k < kN)
      gB[tok * kN + k] = s;
    else
      gC[tok * kN + k - kN] = s;
    return;
  }
  const int64_t j = i - n_bc;
  if (j < d * kN) {
    float s = 0.0f;
    for (int64_t bb = 0; bb < n_ad; ++bb) s += part_a[bb * d * kN + j];
    gA_log[j] = s * -expf(A_log[j]);  // dA/dA_log = A
    return;
  }
  const int64_t c = j - d * kN;
  if (c < d) {
    float s = 0.0f;
    for (int64_t bb = 0; bb < n_ad; ++bb) s += part_d[bb * d + c];
    gD[c] = s;
  }
}

struct BwdWs {
  float* ckpt;
  float* part_bc;
  float* part_a;
  float* part_d;
  float* f_end;
  float* r_out;
  float* s_sum;
  size_t bytes;
  int64_t n_rows;
  int P;
};

BwdWs bwd_layout(int64_t B, int64_t L, int64_t d, char* base) {
  BwdWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off = align256(off + n);
    return base ? reinterpret_cast<float*>(base + o) : nullptr;
  };
  const int64_t nck = (L + kCk - 1) / kCk;
  const int64_t n_tiles = (d + kBwdThreads - 1) / kBwdThreads;
  w.n_rows = n_tiles * 4;
  w.P = bwd_parts(B, L, d);
  const size_t rows = (size_t)w.P * B * d;
  take(sizeof(ErrFlags));  // the error header jm_poll_error reads (cleared each call)
  w.ckpt = take((size_t)B * nck * d * kN * 4);
  w.part_bc = take((size_t)w.n_rows * B * L * 32 * 4);
  w.part_a = take(rows * kN * 4);
  w.part_d = take(rows * 4);
  w.f_end = take(rows * kN * 4);
  w.r_out = take(rows * kN * 4);
  w.s_sum = take(rows * 4);
  w.bytes = off;
  return w;
}

jm_status check_bwd_dims(const jm_dims* dm) {
  if (!dm) {
    set_error("dims is NULL");
    return JM_ERR_INVALID_ARG;
  }
  if (dm->batch < 0 || dm->seqlen < 0 || dm->d_inner <= 0) {
    set_error("sizes must be positive (batch, seqlen >= 0)");
    return JM_ERR_INVALID_ARG;
  }
  if (dm->d_state != kN) {
    set_error("only d_state == 16 is built (got %lld)", (long long)dm->d_state);
    return JM_ERR_UNSUPPORTED;
  }
  if (dm->discretization != JM_DISC_EULER) {
    set_error("the scan backward is built for Euler B (delta B) only");
    return JM_ERR_UNSUPPORTED;
  }
  if (dm->batch > 65535) {
    set_error("batch above 65535 is not supported by the scan backward's launch grid");
    return JM_ERR_INVALID_ARG;
  }
  if ((double)dm->batch * (double)dm->seqlen * (double)dm->d_inner > 1.0e13) {
    set_error("problem too large");
    return JM_ERR_INVALID_ARG;
  }
  return JM_OK;
}

}  // namespace
}  // namespace jmix

using namespace jmix;

JM_API jm_status jm_scan_bwd_schedule(const jm_dims* dims, int* n_parts) {
  if (!n_parts) {
    set_error("jm_scan_bwd_schedule: NULL output pointer");
    return JM_ERR_INVALID_ARG;
  }
  const jm_status st = check_bwd_dims(dims);
  if (st != JM_OK) return st;
  *n_parts = bwd_parts(dims->batch, dims->seqlen, dims->d_inner);
  return JM_OK;
}

JM_API size_t jm_scan_bwd_workspace_size(const jm_dims* dims) {
  if (check_bwd_dims(dims) != JM_OK) return 0;
  return bwd_layout(dims->batch, dims->seqlen, dims->d_inner, nullptr).bytes;
}

JM_API jm_status jm_scan_bwd(const jm_dims* dims, const float* delta, const float* u,
                             const float* Bm, const float* Cm, const float* A_log, const float* D,
                             const float* h0, const float* gy, float* g_delta, float* g_u,
                             float* g_B, float* g_C, float* g_A_log, float* g_D, float* g_h0,
                             void* workspace, size_t ws_bytes, jm_stream_t stream) {
  jm_status st = check_bwd_dims(dims);
  if (st != JM_OK) return st;
  const int64_t B = dims->batch, L = dims->seqlen, d = dims->d_inner;
  const bool any = B > 0 && L > 0;
  const void* const req[] = {A_log, D, g_A_log, g_D};
  const char* const rn[] = {"A_log", "D", "g_A_log", "g_D"};
  for (int i = 0; i < 4; ++i)
    if (!req[i]) {
      set_error("%s is NULL", rn[i]);
      return JM_ERR_INVALID_ARG;
    }
  if (any) {
    const void* const act[] = {delta, u, Bm, Cm, gy, g_delta, g_u, g_B, g_C};
    const char* const an[] = {"delta", "u", "B", "C", "gy", "g_delta", "g_u", "g_B", "g_C"};
    for (int i = 0; i < 9; ++i)
      if (!act[i]) {
        set_error("%s is NULL", an[i]);
        return JM_ERR_INVALID_ARG;
      }
  }
  const size_t need = jm_scan_bwd_workspace_size(dims);
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || ws_bytes < need) {
    set_error("workspace must be 256-byte aligned and at least %zu bytes", need);
    return JM_ERR_WORKSPACE;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(ErrFlags), s);
  if (e != cudaSuccess) {
    // reported below
  } else if (!any) {
    // nothing flows back: every gradient is zero
    e = cudaMemsetAsync(g_A_log, 0, (size_t)d * kN * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g_D, 0, (size_t)d * 4, s);
    if (e == cudaSuccess && g_h0 && B > 0) e = cudaMemsetAsync(g_h0, 0, (size_t)B * d * kN * 4, s);
  } else {
    BwdWs w = bwd_layout(B, L, d, static_cast<char*>(workspace));
    BwdArgs a{B,          L,          d,       delta,   u,       Bm,      Cm,
              A_log,      D,          h0,      gy,      g_delta, g_u,     g_h0,
              w.ckpt,     w.part_bc,  w.part_a, w.part_d, w.P,    w.f_end, w.r_out,
              w.s_sum};
    const dim3 grid((unsigned)((d + kBwdThreads - 1) / kBwdThreads), (unsigned)B, (unsigned)w.P);
    if (w.P > 1) k_scan_bwd_parts<<<grid, kBwdThreads, 0, s>>>(a);
    k_scan_bwd<<<grid, kBwdThreads, 0, s>>>(a);
    const int64_t total = B * L * 32 + d * kN + d;
    k_scan_bwd_reduce<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
        w.part_bc, w.n_rows, B * L, w.part_a, w.part_d, A_log, (int64_t)w.P * B, d, g_B, g_C,
        g_A_log, g_D);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    set_error("CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  return JM_OK;
}
