// fp64 CPU oracle of the Jamba Mamba-1 mixer core.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline / reference legs of bench.py may load this library.  It shares
// no code, header, table or helper with the CUDA path (libjmix).
//
// What it computes (all in double precision, inputs converted exactly):
//   1. causal depthwise conv1d, width K, + SiLU:
//        xc[t,c] = conv_b[c] + sum_{k=0}^{K-1} conv_w[c,k] * X(t-(K-1)+k, c)
//        X(tau,c) = x[tau,c] for tau >= 0, else the cached history
//        init_conv[c, K-1+tau] (or 0); u = xc / (1 + exp(-xc)).
//      (TransformerLens "Jamba" adapter page: the mixer is Mamba-1 with
//       in_proj / conv1d / x_proj / dt_proj / out_proj; width 4 from the
//       llm-architectures-explained "Jamba v0.1" table, mamba_d_conv.)
//   2. x_proj: p[t,j] = sum_c W_x[j,c] u[t,c]; dt = p[0:R], B = p[R:R+N],
//      C = p[R+N:R+2N].
//   3. Jamba's RMSNorms on the selective parameters (TransformerLens adapter
//      page: dt_layernorm / b_layernorm / c_layernorm; RMSNorm of Zhang &
//      Sennrich, NeurIPS 2019, in the Jamba paper's reference list):
//        v_n = v / sqrt(mean(v^2) + eps) * w.
//   4. dt_proj + softplus (aifetchly guide, "Hands-On Implementation":
//      delta = softplus(dt_proj(dt))):
//        delta[t,c] = softplus(sum_r W_dt[c,r] dt_n[t,r] + dt_bias[c]),
//        softplus(v) = max(v,0) + log1p(exp(-|v|)).
//   5. selective scan (aifetchly guide, "Inside the Mamba State-Space Layers",
//      discretisation Abar = exp(delta A), Bbar ~ delta B, and the recurrence
//      h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t h_t), A = -exp(A_log):
//        h[c,n] <- exp(delta[t,c] A[c,n]) h[c,n] + delta[t,c] B[t,n] u[t,c]
//        ys[t,c] = sum_n C[t,n] h[c,n] + D[c] u[t,c]
//   6. gate: y = ys * z / (1 + exp(-z)).  Final SSM state = h after the last
//      token; final conv state = the last K-1 conv inputs, oldest first.
//
// Discretisation of B (orc_dims.zoh): 0 = Euler, Bbar = delta B (the guide's
// "Bbar ~ delta B"); 1 = zero-order hold, Bbar = (exp(delta A) - 1) / A * B,
// the exact one-step solution of dh/dt = A h + B u for u held over the step
// (the guide's continuous-time form, "Selective State Space Model (S6) Forward
// Flow"), taken here as expm1(delta A) / A.
//
// Mirror mode (mirror_bf16 = 1) rounds where the bf16-io CUDA path quantises
// an intermediate: the two tensor-core operands, u as the x_proj operand and
// dt_n as the dt_proj operand, both stored as IEEE fp16.  The rounding is taken
// in the kernel's precision: to float32 (nearest even), then to fp16 (nearest
// even).  The scan uses the unrounded u.  Nothing else is rounded.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

int pick_threads(int32_t t) {
  if (t > 0) return t;
  unsigned h = std::thread::hardware_concurrency();
  return h ? (int)h : 1;
}

// Runs body(i) for i in [0, n) on `threads` threads, contiguous ranges.
template <class F>
void parallel_for(int64_t n, int threads, F body) {
  if (n <= 0) return;
  if (threads <= 1 || n == 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  int64_t nt = std::min<int64_t>(threads, n);
  int64_t per = (n + nt - 1) / nt;
  std::vector<std::thread> pool;
  for (int64_t k = 1; k < nt; ++k) {
    int64_t lo = k * per, hi = std::min(n, lo + per);
    if (lo >= hi) break;
    pool.emplace_back([=] { for (int64_t i = lo; i < hi; ++i) body(i); });
  }
  for (int64_t i = 0; i < std::min(n, per); ++i) body(i);
  for (auto& th : pool) th.join();
}

double round_bf16(double v) {
  float f = (float)v;  // nearest even
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// float32 (nearest even), then IEEE binary16 (nearest even, subnormals kept).
double round_fp16(double v) {
  float f = (float)v;
  _Float16 h = (_Float16)f;
  return (double)(float)h;
}

double silu(double v) { return v / (1.0 + std::exp(-v)); }

// Exact value of element i of a stored input: kind 0 = double, 1 = bf16 bit
// pattern (uint16), 2 = float32.  (Input marshalling only.)
struct Stored {
  const void* p;
  int32_t kind;
  double operator[](int64_t i) const {
    if (kind == 1) {
      uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
      float f;
      std::memcpy(&f, &u, 4);
      return (double)f;
    }
    if (kind == 2) return (double)((const float*)p)[i];
    return ((const double*)p)[i];
  }
};

double softplus(double v) { return std::max(v, 0.0) + std::log1p(std::exp(-std::fabs(v))); }

// The factor that multiplies B u in the state update (see zoh above).
double bbar(double dl, double A, int32_t zoh) { return zoh ? std::expm1(dl * A) / A : dl; }

}  // namespace

extern "C" {

typedef struct {
  int64_t batch, seqlen, d_inner, d_state, d_conv, dt_rank;
  double eps;
  int32_t mirror_bf16;
  int32_t threads;
  int32_t zoh;      // 0: Bbar = delta B; 1: Bbar = expm1(delta A) / A * B
  int32_t reserved;
} orc_dims;

double orc_round_bf16(double v) { return round_bf16(v); }
double orc_round_fp16(double v) { return round_fp16(v); }
double orc_softplus1(double v) { return softplus(v); }

// Step 1 for one sequence: xc [L,d] (pre-activation) from x [L,d].
void orc_conv(int64_t L, int64_t d, int64_t K, const double* x, const double* w,
              const double* b, const double* hist, double* xc) {
  for (int64_t t = 0; t < L; ++t)
    for (int64_t c = 0; c < d; ++c) {
      double acc = b[c];
      for (int64_t k = 0; k < K; ++k) {
        int64_t tau = t - (K - 1) + k;
        double xv = tau >= 0 ? x[tau * d + c] : (hist ? hist[c * (K - 1) + (K - 1) + tau] : 0.0);
        acc += w[c * K + k] * xv;
      }
      xc[t * d + c] = acc;
    }
}

void orc_silu(int64_t n, const double* in, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu(in[i]);
}

void orc_softplus(int64_t n, const double* in, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = softplus(in[i]);
}

// Step 3: RMSNorm of `rows` vectors of length `width` (row stride in_stride).
void orc_rmsnorm(int64_t rows, int64_t width, int64_t in_stride, const double* in,
                 const double* w, double eps, double* out) {
  for (int64_t i = 0; i < rows; ++i) {
    const double* v = in + i * in_stride;
    double ss = 0.0;
    for (int64_t j = 0; j < width; ++j) ss += v[j] * v[j];
    double inv = 1.0 / std::sqrt(ss / (double)width + eps);
    for (int64_t j = 0; j < width; ++j) out[i * width + j] = v[j] * inv * w[j];
  }
}

// Step 5 for one sequence and channels [c0, c1): the recurrence and y_s.
// delta, u: [L,d]; A: [d,N] (already -exp(A_log)); Bm, Cm: [L,N]; h0, hT: [d,N].
void orc_scan_range(int64_t L, int64_t d, int64_t N, const double* delta, const double* A,
                    const double* Bm, const double* Cm, const double* u, const double* D,
                    const double* h0, double* y, double* hT, int64_t c0, int64_t c1,
                    int32_t zoh) {
  std::vector<double> h(N);
  for (int64_t c = c0; c < c1; ++c) {
    for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[c * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      double dl = delta[t * d + c], uv = u[t * d + c];
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const double a = A[c * N + n];
        h[n] = std::exp(dl * a) * h[n] + bbar(dl, a, zoh) * Bm[t * N + n] * uv;
        acc += Cm[t * N + n] * h[n];
      }
      y[t * d + c] = acc + D[c] * uv;
    }
    if (hT)
      for (int64_t n = 0; n < N; ++n) hT[c * N + n] = h[n];
  }
}

void orc_scan(int64_t L, int64_t d, int64_t N, const double* delta, const double* A,
              const double* Bm, const double* Cm, const double* u, const double* D,
              const double* h0, double* y, double* hT, int32_t zoh) {
  orc_scan_range(L, d, N, delta, A, Bm, Cm, u, D, h0, y, hT, 0, d, zoh);
}

// Backward of the scan core of one sequence (Euler B): given gy = dLoss/dy_s
// [L,d], the gradients of delta, u [L,d], B, C [L,N] (summed over channels),
// A [d,N] and D [d] (accumulated: += into gA, gD) and h0 [d,N].  Reverse mode
// of h_t = a_t h_{t-1} + delta_t B_t u_t, a_t = exp(delta_t A), y_t = C_t.h_t +
// D u_t, with every h_t of the forward kept (fp64, small inputs).
void orc_scan_bwd(int64_t L, int64_t d, int64_t N, const double* delta, const double* A,
                  const double* Bm, const double* Cm, const double* u, const double* D,
                  const double* h0, const double* gy, double* gdelta, double* gu, double* gB,
                  double* gC, double* gA, double* gD, double* gh0) {
  for (int64_t i = 0; i < L * N; ++i) gB[i] = gC[i] = 0.0;
  std::vector<double> hs((size_t)(L + 1) * N), g(N);
  for (int64_t c = 0; c < d; ++c) {
    for (int64_t n = 0; n < N; ++n) hs[n] = h0 ? h0[c * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      const double dl = delta[t * d + c], uv = u[t * d + c];
      for (int64_t n = 0; n < N; ++n)
        hs[(t + 1) * N + n] = std::exp(dl * A[c * N + n]) * hs[t * N + n] + dl * Bm[t * N + n] * uv;
    }
    for (int64_t n = 0; n < N; ++n) g[n] = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
      const double dl = delta[t * d + c], uv = u[t * d + c], gyt = gy[t * d + c];
      double gdl = 0.0, gut = D[c] * gyt;
      gD[c] += gyt * uv;
      for (int64_t n = 0; n < N; ++n) {
        const double a = std::exp(dl * A[c * N + n]);
        const double hp = hs[t * N + n], ht = hs[(t + 1) * N + n];
        g[n] += Cm[t * N + n] * gyt;             // y_t = C_t . h_t + ...
        gC[t * N + n] += gyt * ht;
        gut += g[n] * dl * Bm[t * N + n];
        gB[t * N + n] += g[n] * dl * uv;
        gdl += g[n] * (A[c * N + n] * a * hp + Bm[t * N + n] * uv);
        gA[c * N + n] += g[n] * dl * a * hp;
        g[n] *= a;                               // to h_{t-1}
      }
      gdelta[t * d + c] = gdl;
      gu[t * d + c] = gut;
    }
    if (gh0)
      for (int64_t n = 0; n < N; ++n) gh0[c * N + n] = g[n];
  }
}

// Front end of one sequence for tokens [t0, t1): u, p rows (from the
// mirror-rounded u in mirror mode), normalised dt_n (mirror-rounded) / Bn / Cn.
static void front_end_rows(const orc_dims* m, Stored x, const double* conv_w,
                           const double* conv_b, const double* xproj_wT /*[d,P]*/,
                           const double* dtn_w, const double* bn_w, const double* cn_w,
                           const double* hist, int64_t t0, int64_t t1, double* u_rows /*[t1-t0,d]*/,
                           double* dtn /*[L,R]*/, double* Bn /*[L,N]*/, double* Cn /*[L,N]*/) {
  const int64_t d = m->d_inner, K = m->d_conv, N = m->d_state, R = m->dt_rank, P = R + 2 * N;
  std::vector<double> p(P);
  for (int64_t t = t0; t < t1; ++t) {
    double* ur = u_rows + (t - t0) * d;
    for (int64_t c = 0; c < d; ++c) {
      double acc = conv_b[c];
      for (int64_t k = 0; k < K; ++k) {
        int64_t tau = t - (K - 1) + k;
        double xv = tau >= 0 ? x[tau * d + c] : (hist ? hist[c * (K - 1) + (K - 1) + tau] : 0.0);
        acc += conv_w[c * K + k] * xv;
      }
      ur[c] = silu(acc);
    }
    // p[j] = sum_c W_x[j,c] u[c], summed in ascending c for every j
    std::fill(p.begin(), p.end(), 0.0);
    for (int64_t c = 0; c < d; ++c) {
      const double uc = m->mirror_bf16 ? round_fp16(ur[c]) : ur[c];
      const double* wr = xproj_wT + c * P;
      for (int64_t j = 0; j < P; ++j) p[j] += wr[j] * uc;
    }
    orc_rmsnorm(1, R, R, p.data(), dtn_w, m->eps, dtn + t * R);
    orc_rmsnorm(1, N, N, p.data() + R, bn_w, m->eps, Bn + t * N);
    orc_rmsnorm(1, N, N, p.data() + R + N, cn_w, m->eps, Cn + t * N);
    if (m->mirror_bf16)
      for (int64_t r = 0; r < R; ++r) dtn[t * R + r] = round_fp16(dtn[t * R + r]);
  }
}

static std::vector<double> transpose(const double* a, int64_t rows, int64_t cols) {
  std::vector<double> t((size_t)rows * cols);
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t j = 0; j < cols; ++j) t[j * rows + i] = a[i * cols + j];
  return t;
}

// delta for channels ch[0..nch) of one sequence: out [L, nch].
static void dt_proj_channels(const orc_dims* m, const double* dtn, const double* dtproj_w,
                             const double* dt_bias, int64_t L, int64_t nch, const int64_t* ch,
                             double* out, int threads) {
  const int64_t R = m->dt_rank;
  parallel_for(L, threads, [&](int64_t t) {
    for (int64_t i = 0; i < nch; ++i) {
      const double* wr = dtproj_w + ch[i] * R;
      double acc = 0.0;
      for (int64_t r = 0; r < R; ++r) acc += wr[r] * dtn[t * R + r];
      out[t * nch + i] = softplus(acc + dt_bias[ch[i]]);
    }
  });
}

// The whole mixer forward for the channels ch[0..nch) of every sequence.  The
// front end (conv, x_proj, norms) runs over all channels, since B, C and dt
// depend on all of them; dt_proj, the scan and the gate run only for ch.
// x: [B, L, d] stored as x_kind (see Stored); z_sel: [B, L, nch], the z values
// of the chosen channels.  y: [B, L, nch]; final_state: [B, nch, N] (or null);
// final_conv: [B, nch, K-1] (or null).
void orc_mixer_fwd_channels(const orc_dims* m, const void* x_data, int32_t x_kind,
                            const double* z_sel,
                            const double* conv_w, const double* conv_b, const double* xproj_w,
                            const double* dtn_w, const double* bn_w, const double* cn_w,
                            const double* dtproj_w, const double* dt_bias, const double* A_log,
                            const double* D, const double* init_conv, const double* init_ssm,
                            int64_t nch, const int64_t* ch, double* y, double* final_state,
                            double* final_conv) {
  const int64_t Bt = m->batch, L = m->seqlen, d = m->d_inner, N = m->d_state, K = m->d_conv,
                R = m->dt_rank, P = R + 2 * N;
  const int threads = pick_threads(m->threads);
  std::vector<double> wT = transpose(xproj_w, P, d);
  std::vector<double> dtn((size_t)L * R), Bn((size_t)L * N), Cn((size_t)L * N);
  std::vector<double> usel((size_t)L * nch), delta((size_t)L * nch);
  const int64_t blk = 64;
  const int64_t nblk = (L + blk - 1) / blk;
  for (int64_t b = 0; b < Bt; ++b) {
    const Stored xb{x_kind == 1   ? (const void*)((const uint16_t*)x_data + b * L * d)
                    : x_kind == 2 ? (const void*)((const float*)x_data + b * L * d)
                                  : (const void*)((const double*)x_data + b * L * d),
                    x_kind};
    const double* hist = init_conv ? init_conv + b * d * (K - 1) : nullptr;
    parallel_for(nblk, threads, [&](int64_t ib) {
      int64_t t0 = ib * blk, t1 = std::min(L, t0 + blk);
      std::vector<double> ur((size_t)(t1 - t0) * d);
      front_end_rows(m, xb, conv_w, conv_b, wT.data(), dtn_w, bn_w, cn_w, hist, t0, t1, ur.data(),
                     dtn.data(), Bn.data(), Cn.data());
      for (int64_t t = t0; t < t1; ++t)
        for (int64_t i = 0; i < nch; ++i) usel[t * nch + i] = ur[(t - t0) * d + ch[i]];
    });
    dt_proj_channels(m, dtn.data(), dtproj_w, dt_bias, L, nch, ch, delta.data(), threads);
    parallel_for(nch, threads, [&](int64_t i) {
      const int64_t c = ch[i];
      std::vector<double> h(N), A(N);
      for (int64_t n = 0; n < N; ++n) {
        A[n] = -std::exp(A_log[c * N + n]);
        h[n] = init_ssm ? init_ssm[(b * d + c) * N + n] : 0.0;
      }
      for (int64_t t = 0; t < L; ++t) {
        double dl = delta[t * nch + i], uv = usel[t * nch + i];
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          h[n] = std::exp(dl * A[n]) * h[n] + bbar(dl, A[n], m->zoh) * Bn[t * N + n] * uv;
          acc += Cn[t * N + n] * h[n];
        }
        double ys = acc + D[c] * uv;
        y[(b * L + t) * nch + i] = ys * silu(z_sel[(b * L + t) * nch + i]);
      }
      if (final_state)
        for (int64_t n = 0; n < N; ++n) final_state[(b * nch + i) * N + n] = h[n];
      if (final_conv)
        for (int64_t k = 0; k < K - 1; ++k) {
          int64_t tau = L - (K - 1) + k;
          final_conv[(b * nch + i) * (K - 1) + k] =
              tau >= 0 ? xb[tau * d + c] : (hist ? hist[c * (K - 1) + (K - 1) + tau] : 0.0);
        }
    });
  }
}

// The whole mixer forward over all channels.
// y: [B,L,d]; final_state: [B,d,N]; final_conv: [B,d,K-1] (each may be null).
void orc_mixer_fwd(const orc_dims* m, const double* x, const double* z, const double* conv_w,
                   const double* conv_b, const double* xproj_w, const double* dtn_w,
                   const double* bn_w, const double* cn_w, const double* dtproj_w,
                   const double* dt_bias, const double* A_log, const double* D,
                   const double* init_conv, const double* init_ssm, double* y,
                   double* final_state, double* final_conv) {
  std::vector<int64_t> ch(m->d_inner);
  for (int64_t c = 0; c < m->d_inner; ++c) ch[c] = c;
  orc_mixer_fwd_channels(m, x, 0, z, conv_w, conv_b, xproj_w, dtn_w, bn_w, cn_w, dtproj_w,
                         dt_bias, A_log, D, init_conv, init_ssm, m->d_inner, ch.data(), y,
                         final_state, final_conv);
}

// One decode step for every sequence: the forward with L = 1 and the cached
// states as history, then conv_state <- [s_1 .. s_{K-2}, x_t] and
// ssm_state <- h (both in place).  x_t, z_t, y_t: [B,d].
void orc_mixer_step(const orc_dims* m, const double* x_t, const double* z_t, double* conv_state,
                    double* ssm_state, const double* conv_w, const double* conv_b,
                    const double* xproj_w, const double* dtn_w, const double* bn_w,
                    const double* cn_w, const double* dtproj_w, const double* dt_bias,
                    const double* A_log, const double* D, double* y_t) {
  orc_dims one = *m;
  one.seqlen = 1;
  const int64_t Bt = m->batch, d = m->d_inner, N = m->d_state, K = m->d_conv;
  std::vector<double> fs((size_t)d * N), fc((size_t)d * (K - 1));
  for (int64_t b = 0; b < Bt; ++b) {
    one.batch = 1;
    orc_mixer_fwd(&one, x_t + b * d, z_t + b * d, conv_w, conv_b, xproj_w, dtn_w, bn_w, cn_w,
                  dtproj_w, dt_bias, A_log, D, conv_state + b * d * (K - 1), ssm_state + b * d * N,
                  y_t + b * d, fs.data(), fc.data());
    std::memcpy(ssm_state + b * d * N, fs.data(), sizeof(double) * d * N);
    std::memcpy(conv_state + b * d * (K - 1), fc.data(), sizeof(double) * d * (K - 1));
  }
}

}  // extern "C"
