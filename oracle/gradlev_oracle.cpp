// GradLev scan oracle: plain, serial, float64 CPU implementation.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and
// its Python binding) may include, link or call this file; only the tests,
// the package's smoke check and the CPU-baseline leg of the benchmark do.
// It shares no code, header or constant with the CUDA path.
//
// What it computes (one adaptive linear layer, per batch b and head h):
//
//   Cognaptus, "Parallelize the Training, Keep the Learning Serial", section
//   "Once the gradient signals are known, the weight trajectory becomes
//   parallelizable": a temporary weight W_t, initialised from the persistent
//   weight W_0, is updated once per token with a centred rule driven by the
//   layer input x_t, a step size eta_t, a retention gate alpha_t and the
//   costate g_t (gradient of the token loss w.r.t. the layer output). The
//   display equation is missing from the extracted page; the reading used here
//   (the deviation D = W - W_0 decays by alpha and receives a rank-one
//   gradient step) is:
//
//       D_0 = 0,   y_t = (W_0 + D_{t-1}) x_t,   D_t = alpha_t D_{t-1} - eta_t g_t x_t^T
//
//   in the page's 1-based notation. With 0-based tokens and S_t := the
//   deviation BEFORE token t this is
//
//       S_0 = 0,   y_t = (W_0 + S_t) x_t,       S_{t+1} = alpha_t S_t - eta_t g_t x_t^T.
//
//   GradLev abstract (omanscience.com / scholarbro.com, "GradLev: Token-Parallel
//   Test-Time Training Via Costate Prediction", Abstract): given inputs and
//   costates, online gradient descent admits exact scans for forward
//   evaluation and for reverse backpropagation. The backward here is the exact
//   reverse-mode derivative of the recurrence above for the scalar objective
//   L = sum_t <u_t, y_t> (u = dL/dy supplied by the caller), written as the
//   adjoint recurrence of the state:
//
//       Lam_T = 0,   Lam_t = dL/dS_t = alpha_t Lam_{t+1} + u_t x_t^T
//       dx_t     = (W_0 + S_t)^T u_t - eta_t Lam_{t+1}^T g_t
//       dg_t     = -eta_t Lam_{t+1} x_t
//       deta_t   = -g_t . (Lam_{t+1} x_t)
//       dalpha_t = <Lam_{t+1}, S_t>_F
//       dW_0     = sum over b and t of u_t x_t^T      (W_0 is one matrix per head)
//
// Carried state (a sequence split across calls). The same section notes that
// the recurrence is affine, so partial results combine: the second part of a
// split sequence continues from the deviation the first part left. The
// streaming entry points take that start deviation S_0 (zero for a fresh
// sequence) and return the end deviation S_T; in reverse they take the
// objective's gradient with respect to S_T (Lam_T, the adjoint flowing in
// from the later part) and return dL/dS_0:
//
//       L = sum_t <u_t, y_t> + <Lam_T, S_T>_F,   dS_0 = Lam_0
//
// with the adjoint recurrence above started from that Lam_T. Every other
// output keeps its formula, with S_t now including the carried S_0.
//
// Everything is materialised token by token in double (or complex<double> for
// the complex-step derivative checks); there is no chunking, no blocking and
// no reordering beyond this serial definition. OpenMP is used only across the
// independent (b, h) pairs; the token loop of each pair is serial.
//
// Layouts (row-major, contiguous):
//   x, dx [B,H,T,d_in]   g, y, dy, dg [B,H,T,d_out]   eta, alpha, deta, dalpha [B,H,T]
//   W0, dW0 [H,d_out,d_in]   (dW0 is summed over b in a fixed order b = 0..B-1)

#include <cmath>
#include <complex>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

using cplx = std::complex<double>;

inline size_t at3(int b, int h, int t, int H, int T) {
  return ((size_t)b * H + h) * (size_t)T + t;
}

// S <- alpha S - eta g x^T
template <class R>
void state_step(int din, int dout, R* S, R alpha, R eta, const R* g, const R* x) {
  for (int n = 0; n < dout; ++n)
    for (int k = 0; k < din; ++k)
      S[(size_t)n * din + k] = alpha * S[(size_t)n * din + k] - eta * g[n] * x[k];
}

// Forward of one (b,h) scan. S_work holds d_out*d_in scalars. S0 (or null for
// zero) is the start deviation; if S_traj is non-null it receives S_0 .. S_T
// ((T+1)*d_out*d_in scalars); if ST is non-null it receives S_T.
template <class R>
void fwd_head(int T, int din, int dout, const R* x, const R* g, const R* eta,
              const R* alpha, const R* W0, R* y, R* S_work, R* S_traj,
              const R* S0 = nullptr, R* ST = nullptr) {
  const size_t dd = (size_t)din * dout;
  for (size_t e = 0; e < dd; ++e) S_work[e] = S0 ? S0[e] : R(0);
  if (S_traj) std::memcpy(S_traj, S_work, dd * sizeof(R));
  for (int t = 0; t < T; ++t) {
    const R* xt = x + (size_t)t * din;
    for (int n = 0; n < dout; ++n) {
      R acc(0);
      for (int k = 0; k < din; ++k)
        acc += (W0[(size_t)n * din + k] + S_work[(size_t)n * din + k]) * xt[k];
      y[(size_t)t * dout + n] = acc;
    }
    state_step(din, dout, S_work, alpha[t], eta[t], g + (size_t)t * dout, xt);
    if (S_traj) std::memcpy(S_traj + (size_t)(t + 1) * dd, S_work, dd * sizeof(R));
  }
  if (ST) std::memcpy(ST, S_work, dd * sizeof(R));
}

// Backward of one (b,h) scan. S_t is needed in reverse order; the forward
// sweep stores S at every `ckpt`-th token and each segment is re-run forward
// from its checkpoint before it is walked backwards. dW0p receives this pair's
// sum_t u_t x_t^T. `mutate` = 1 replaces (W_0 + S_t)^T by W_0^T in dx: the
// negative control of the "synthetic test" section (persistent instead of
// adapted weight in the backward reconstruction), used only by tests.
// S0 / LamT (null for zero): the carried start deviation and the adjoint
// flowing in at the end; dS0 (if non-null) receives Lam_0.
void bwd_head(int T, int din, int dout, const double* x, const double* g,
              const double* eta, const double* alpha, const double* W0,
              const double* u, double* dx, double* dg, double* deta,
              double* dalpha, double* dW0p, int ckpt, int mutate,
              const double* S0 = nullptr, const double* LamT = nullptr,
              double* dS0 = nullptr) {
  const size_t dd = (size_t)din * dout;
  if (ckpt < 1) ckpt = 1;
  const int nseg = (T + ckpt - 1) / ckpt;
  std::vector<double> ck((size_t)nseg * dd, 0.0);
  std::vector<double> S(dd, 0.0);
  if (S0) std::memcpy(S.data(), S0, dd * sizeof(double));
  for (int t = 0; t < T; ++t) {
    if (t % ckpt == 0) std::memcpy(&ck[(size_t)(t / ckpt) * dd], S.data(), dd * sizeof(double));
    state_step(din, dout, S.data(), alpha[t], eta[t], g + (size_t)t * dout, x + (size_t)t * din);
  }
  std::vector<double> seg((size_t)ckpt * dd);
  std::vector<double> Lam(dd, 0.0), r(dout);
  if (LamT) std::memcpy(Lam.data(), LamT, dd * sizeof(double));
  for (size_t e = 0; e < dd; ++e) dW0p[e] = 0.0;
  for (int s = nseg - 1; s >= 0; --s) {
    const int t0 = s * ckpt, t1 = (t0 + ckpt < T) ? t0 + ckpt : T;
    std::memcpy(S.data(), &ck[(size_t)s * dd], dd * sizeof(double));
    for (int t = t0; t < t1; ++t) {
      std::memcpy(&seg[(size_t)(t - t0) * dd], S.data(), dd * sizeof(double));
      state_step(din, dout, S.data(), alpha[t], eta[t], g + (size_t)t * dout, x + (size_t)t * din);
    }
    for (int t = t1 - 1; t >= t0; --t) {
      const double* St = &seg[(size_t)(t - t0) * dd];  // S_t
      const double* xt = x + (size_t)t * din;
      const double* gt = g + (size_t)t * dout;
      const double* ut = u + (size_t)t * dout;
      // Lam currently holds Lam_{t+1}.
      for (int n = 0; n < dout; ++n) {
        double acc = 0.0;
        for (int k = 0; k < din; ++k) acc += Lam[(size_t)n * din + k] * xt[k];
        r[n] = acc;
      }
      double ge = 0.0;
      for (int n = 0; n < dout; ++n) {
        dg[(size_t)t * dout + n] = -eta[t] * r[n];
        ge += gt[n] * r[n];
      }
      deta[t] = -ge;
      double ip = 0.0;
      for (size_t e = 0; e < dd; ++e) ip += Lam[e] * St[e];
      dalpha[t] = ip;
      for (int k = 0; k < din; ++k) {
        double acc = 0.0;
        for (int n = 0; n < dout; ++n) {
          const double w = mutate ? W0[(size_t)n * din + k]
                                  : W0[(size_t)n * din + k] + St[(size_t)n * din + k];
          acc += w * ut[n] - eta[t] * Lam[(size_t)n * din + k] * gt[n];
        }
        dx[(size_t)t * din + k] = acc;
      }
      for (int n = 0; n < dout; ++n)
        for (int k = 0; k < din; ++k) {
          dW0p[(size_t)n * din + k] += ut[n] * xt[k];
          Lam[(size_t)n * din + k] = alpha[t] * Lam[(size_t)n * din + k] + ut[n] * xt[k];
        }
    }
  }
  if (dS0) std::memcpy(dS0, Lam.data(), dd * sizeof(double));
}

// Serial online learner with inner loss 0.5 ||W x_t - v_t||^2 (the learner
// GradLev is meant to recover; "The predictor is constrained by the learner it
// is supposed to reproduce"): y_t = W x_t, g*_t = y_t - v_t, then the same
// centred update W <- W_0 + alpha_t (W - W_0) - eta_t g*_t x_t^T.
template <class R>
void serial_head(int T, int din, int dout, const R* x, const R* v, const R* eta,
                 const R* alpha, const R* W0, R* y, R* gstar) {
  const size_t dd = (size_t)din * dout;
  std::vector<R> W(W0, W0 + dd);
  for (int t = 0; t < T; ++t) {
    const R* xt = x + (size_t)t * din;
    for (int n = 0; n < dout; ++n) {
      R acc(0);
      for (int k = 0; k < din; ++k) acc += W[(size_t)n * din + k] * xt[k];
      y[(size_t)t * dout + n] = acc;
      gstar[(size_t)t * dout + n] = acc - v[(size_t)t * dout + n];
    }
    for (int n = 0; n < dout; ++n)
      for (int k = 0; k < din; ++k) {
        const size_t e = (size_t)n * din + k;
        W[e] = W0[e] + alpha[t] * (W[e] - W0[e]) - eta[t] * gstar[(size_t)t * dout + n] * xt[k];
      }
  }
}

// Deployment decode of one (b,h) pair (GradLev abstract: at deployment the
// auxiliary predictor is discarded and the model updates itself by
// token-by-token forward and backward passes; Cognaptus, same page, opening
// section: deployment still runs a forward pass, a backward pass and a weight
// update per token). For the single adapted layer with the synthetic test's
// inner loss 0.5 ||W x_t - v_t||^2, one token is
//     y_t = (W_0 + S) x_t,   g_t = y_t - v_t,   S <- alpha_t S - eta_t g_t x_t^T
// with S the deviation carried between calls (in/out).
template <class R>
void decode_head(int T, int din, int dout, const R* x, const R* v, const R* eta,
                 const R* alpha, const R* W0, R* S, R* y, R* g) {
  for (int t = 0; t < T; ++t) {
    const R* xt = x + (size_t)t * din;
    for (int n = 0; n < dout; ++n) {
      R acc(0);
      for (int k = 0; k < din; ++k)
        acc += (W0[(size_t)n * din + k] + S[(size_t)n * din + k]) * xt[k];
      y[(size_t)t * dout + n] = acc;
      g[(size_t)t * dout + n] = acc - v[(size_t)t * dout + n];
    }
    state_step(din, dout, S, alpha[t], eta[t], g + (size_t)t * dout, xt);
  }
}

// Two-layer adapted MLP of the synthetic test (Cognaptus, same page, section
// "The synthetic test checks the mechanism, not model quality"). Both matrices
// adapt with the centred rule; the pages do not name the nonlinearity, and tanh
// is used here. Shared gates eta_t, alpha_t drive both layers. Per token:
//   a_t = (W1 + S1) x_t,  h_t = tanh(a_t),  y_t = (W2 + S2) h_t,
//   g2_t = y_t - v_t,     g1_t = (1 - h_t^2) (.) ((W2 + S2)^T g2_t),
//   S1 <- alpha_t S1 - eta_t g1_t x_t^T,  S2 <- alpha_t S2 - eta_t g2_t h_t^T,
// i.e. serial test-time backpropagation of the token loss 0.5 ||y_t - v_t||^2.
// Shapes: x [T,dx], v/y/g2 [T,dy], g1 [T,dh], W1 [dh,dx], W2 [dy,dh].
template <class R>
void mlp2_serial_head(int T, int dx, int dh, int dy, const R* x, const R* v, const R* eta,
                      const R* alpha, const R* W1, const R* W2, R* y, R* g1, R* g2) {
  std::vector<R> S1((size_t)dh * dx, R(0)), S2((size_t)dy * dh, R(0)), a(dh), h(dh), q(dh);
  for (int t = 0; t < T; ++t) {
    const R* xt = x + (size_t)t * dx;
    for (int k = 0; k < dh; ++k) {
      R acc(0);
      for (int m = 0; m < dx; ++m) acc += (W1[(size_t)k * dx + m] + S1[(size_t)k * dx + m]) * xt[m];
      a[k] = acc;
      h[k] = std::tanh(acc);
    }
    R* g2t = g2 + (size_t)t * dy;
    for (int n = 0; n < dy; ++n) {
      R acc(0);
      for (int k = 0; k < dh; ++k) acc += (W2[(size_t)n * dh + k] + S2[(size_t)n * dh + k]) * h[k];
      y[(size_t)t * dy + n] = acc;
      g2t[n] = acc - v[(size_t)t * dy + n];
    }
    R* g1t = g1 + (size_t)t * dh;
    for (int k = 0; k < dh; ++k) {
      R acc(0);
      for (int n = 0; n < dy; ++n) acc += (W2[(size_t)n * dh + k] + S2[(size_t)n * dh + k]) * g2t[n];
      g1t[k] = (R(1) - h[k] * h[k]) * acc;
    }
    state_step(dx, dh, S1.data(), alpha[t], eta[t], g1t, xt);
    state_step(dh, dy, S2.data(), alpha[t], eta[t], g2t, h.data());
  }
}

// The parallel reconstruction of the same two layers from given costates g1hat,
// g2hat, as the pages describe it: both layers' forwards are scans driven by the
// given costates, and the costates the trajectory implies are then reconstructed
// by backpropagating each token's loss through the adapted weights of that token:
//   a = scan(x; g1hat, W1),  h = tanh(a),  y = scan(h; g2hat, W2),
//   g2til_t = y_t - v_t,  g1til_t = (1 - h_t^2) (.) ((W2 + S2_t)^T g2til_t),
//   dW1 = sum_t g1til_t x_t^T   (the first matrix's gradient over the sequence).
// control = 1 replaces the adapted W2 + S2_t by the persistent W2 in the
// reconstruction: the control of the synthetic-test section.
void mlp2_recon_head(int T, int dx, int dh, int dy, const double* x, const double* g1hat,
                     const double* g2hat, const double* v, const double* eta,
                     const double* alpha, const double* W1, const double* W2, int control,
                     double* a, double* h, double* y, double* g2til, double* g1til,
                     double* dW1) {
  std::vector<double> S1((size_t)dh * dx), S2((size_t)dy * dh, 0.0);
  fwd_head<double>(T, dx, dh, x, g1hat, eta, alpha, W1, a, S1.data(), nullptr);
  for (size_t e = 0; e < (size_t)T * dh; ++e) h[e] = std::tanh(a[e]);
  for (size_t e = 0; e < (size_t)dh * dx; ++e) dW1[e] = 0.0;
  for (int t = 0; t < T; ++t) {
    const double* ht = h + (size_t)t * dh;
    double* g2t = g2til + (size_t)t * dy;
    for (int n = 0; n < dy; ++n) {
      double acc = 0.0;
      for (int k = 0; k < dh; ++k) acc += (W2[(size_t)n * dh + k] + S2[(size_t)n * dh + k]) * ht[k];
      y[(size_t)t * dy + n] = acc;
      g2t[n] = acc - v[(size_t)t * dy + n];
    }
    double* g1t = g1til + (size_t)t * dh;
    for (int k = 0; k < dh; ++k) {
      double acc = 0.0;
      for (int n = 0; n < dy; ++n) {
        const double w = control ? W2[(size_t)n * dh + k]
                                 : W2[(size_t)n * dh + k] + S2[(size_t)n * dh + k];
        acc += w * g2t[n];
      }
      g1t[k] = (1.0 - ht[k] * ht[k]) * acc;
      for (int m = 0; m < dx; ++m) dW1[(size_t)k * dx + m] += g1t[k] * x[(size_t)t * dx + m];
    }
    state_step(dh, dy, S2.data(), alpha[t], eta[t], g2hat + (size_t)t * dy, ht);
  }
}

inline int pick_threads(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

// S0, ST: null, or [B,H,d_out,d_in] start / end deviations.
template <class R>
void fwd_all(int B, int H, int T, int din, int dout, const R* x, const R* g, const R* eta,
             const R* alpha, const R* W0, R* y, int nthreads, const R* S0 = nullptr,
             R* ST = nullptr) {
  const int nt = pick_threads(nthreads);
  const size_t dd = (size_t)din * dout;
#pragma omp parallel num_threads(nt)
  {
    std::vector<R> S(dd);
#pragma omp for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
      const int b = bh / H, h = bh % H;
      const size_t o = at3(b, h, 0, H, T);
      fwd_head<R>(T, din, dout, x + o * din, g + o * dout, eta + o, alpha + o,
                  W0 + (size_t)h * dd, y + o * dout, S.data(), nullptr,
                  S0 ? S0 + (size_t)bh * dd : nullptr, ST ? ST + (size_t)bh * dd : nullptr);
    }
  }
}

template <class R>
void serial_all(int B, int H, int T, int din, int dout, const R* x, const R* v, const R* eta,
                const R* alpha, const R* W0, R* y, R* gstar, int nthreads) {
  const int nt = pick_threads(nthreads);
  const size_t dd = (size_t)din * dout;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
    const int b = bh / H, h = bh % H;
    const size_t o = at3(b, h, 0, H, T);
    serial_head<R>(T, din, dout, x + o * din, v + o * dout, eta + o, alpha + o,
                   W0 + (size_t)h * dd, y + o * dout, gstar + o * dout);
  }
}

}  // namespace

extern "C" {

// y = forward scan (see file header). nthreads <= 0: OpenMP default.
void oracle_fwd_f64(int B, int H, int T, int din, int dout, const double* x, const double* g,
                    const double* eta, const double* alpha, const double* W0, double* y,
                    int nthreads) {
  fwd_all<double>(B, H, T, din, dout, x, g, eta, alpha, W0, y, nthreads);
}

// Same in complex arithmetic (arrays are interleaved re,im pairs). Used for
// complex-step derivatives: Im f(a + i h v) / h = <df/da, v> + O(h^2).
void oracle_fwd_c128(int B, int H, int T, int din, int dout, const double* x, const double* g,
                     const double* eta, const double* alpha, const double* W0, double* y,
                     int nthreads) {
  fwd_all<cplx>(B, H, T, din, dout, reinterpret_cast<const cplx*>(x),
                reinterpret_cast<const cplx*>(g), reinterpret_cast<const cplx*>(eta),
                reinterpret_cast<const cplx*>(alpha), reinterpret_cast<const cplx*>(W0),
                reinterpret_cast<cplx*>(y), nthreads);
}

// Forward with the carried state (see file header): S0 may be null (zero), ST
// may be null (not written); both [B,H,d_out,d_in].
void oracle_fwd_state_f64(int B, int H, int T, int din, int dout, const double* x,
                          const double* g, const double* eta, const double* alpha,
                          const double* W0, const double* S0, double* y, double* ST,
                          int nthreads) {
  fwd_all<double>(B, H, T, din, dout, x, g, eta, alpha, W0, y, nthreads, S0, ST);
}

void oracle_fwd_state_c128(int B, int H, int T, int din, int dout, const double* x,
                           const double* g, const double* eta, const double* alpha,
                           const double* W0, const double* S0, double* y, double* ST,
                           int nthreads) {
  fwd_all<cplx>(B, H, T, din, dout, reinterpret_cast<const cplx*>(x),
                reinterpret_cast<const cplx*>(g), reinterpret_cast<const cplx*>(eta),
                reinterpret_cast<const cplx*>(alpha), reinterpret_cast<const cplx*>(W0),
                reinterpret_cast<cplx*>(y), nthreads, reinterpret_cast<const cplx*>(S0),
                reinterpret_cast<cplx*>(ST));
}

// Whole state trajectory S_0..S_T of ONE scan (B = H = 1), for small tests.
void oracle_states_f64(int T, int din, int dout, const double* x, const double* g,
                       const double* eta, const double* alpha, const double* W0, double* y,
                       double* S_traj) {
  std::vector<double> S((size_t)din * dout);
  fwd_head<double>(T, din, dout, x, g, eta, alpha, W0, y, S.data(), S_traj);
}

// Reverse scan (see file header). ckpt: checkpoint interval of the state
// recompute (any value >= 1 gives the same result up to nothing: the recompute
// is the same serial arithmetic). flags bit 0: negative-control mutation.
void oracle_bwd_state_f64(int B, int H, int T, int din, int dout, const double* x,
                          const double* g, const double* eta, const double* alpha,
                          const double* W0, const double* S0, const double* dy,
                          const double* LamT, double* dx, double* dg, double* deta,
                          double* dalpha, double* dW0, double* dS0, int ckpt, int flags,
                          int nthreads);

void oracle_bwd_f64(int B, int H, int T, int din, int dout, const double* x, const double* g,
                    const double* eta, const double* alpha, const double* W0, const double* dy,
                    double* dx, double* dg, double* deta, double* dalpha, double* dW0,
                    int ckpt, int flags, int nthreads) {
  oracle_bwd_state_f64(B, H, T, din, dout, x, g, eta, alpha, W0, nullptr, dy, nullptr, dx, dg,
                       deta, dalpha, dW0, nullptr, ckpt, flags, nthreads);
}

// Reverse scan with the carried state (see file header): S0 and LamT may be null
// (zero), dS0 may be null (not written); all three are [B,H,d_out,d_in].
void oracle_bwd_state_f64(int B, int H, int T, int din, int dout, const double* x,
                          const double* g, const double* eta, const double* alpha,
                          const double* W0, const double* S0, const double* dy,
                          const double* LamT, double* dx, double* dg, double* deta,
                          double* dalpha, double* dW0, double* dS0, int ckpt, int flags,
                          int nthreads) {
  const int nt = pick_threads(nthreads);
  const size_t dd = (size_t)din * dout;
  std::vector<double> part((size_t)B * H * dd);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
    const int b = bh / H, h = bh % H;
    const size_t o = at3(b, h, 0, H, T);
    bwd_head(T, din, dout, x + o * din, g + o * dout, eta + o, alpha + o, W0 + (size_t)h * dd,
             dy + o * dout, dx + o * din, dg + o * dout, deta + o, dalpha + o,
             &part[(size_t)bh * dd], ckpt, flags & 1, S0 ? S0 + (size_t)bh * dd : nullptr,
             LamT ? LamT + (size_t)bh * dd : nullptr, dS0 ? dS0 + (size_t)bh * dd : nullptr);
  }
  for (int h = 0; h < H; ++h) {
    double* out = dW0 + (size_t)h * dd;
    for (size_t e = 0; e < dd; ++e) out[e] = 0.0;
    for (int b = 0; b < B; ++b) {
      const double* p = &part[((size_t)b * H + h) * dd];
      for (size_t e = 0; e < dd; ++e) out[e] += p[e];
    }
  }
}

// Serial online learner (inner loss 0.5||W x - v||^2): outputs y and the true
// serial costates g* = y - v.
void oracle_serial_f64(int B, int H, int T, int din, int dout, const double* x, const double* v,
                       const double* eta, const double* alpha, const double* W0, double* y,
                       double* gstar, int nthreads) {
  serial_all<double>(B, H, T, din, dout, x, v, eta, alpha, W0, y, gstar, nthreads);
}

void oracle_serial_c128(int B, int H, int T, int din, int dout, const double* x, const double* v,
                        const double* eta, const double* alpha, const double* W0, double* y,
                        double* gstar, int nthreads) {
  serial_all<cplx>(B, H, T, din, dout, reinterpret_cast<const cplx*>(x),
                   reinterpret_cast<const cplx*>(v), reinterpret_cast<const cplx*>(eta),
                   reinterpret_cast<const cplx*>(alpha), reinterpret_cast<const cplx*>(W0),
                   reinterpret_cast<cplx*>(y), reinterpret_cast<cplx*>(gstar), nthreads);
}

// Deployment decode of T tokens per pair (see decode_head): S [B,H,d_out,d_in]
// is read and overwritten with the deviation after the last token; y and g
// [B,H,T,d_out] receive the outputs and the costates.
void oracle_decode_f64(int B, int H, int T, int din, int dout, const double* x, const double* v,
                       const double* eta, const double* alpha, const double* W0, double* S,
                       double* y, double* g, int nthreads) {
  const int nt = pick_threads(nthreads);
  const size_t dd = (size_t)din * dout;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
    const int b = bh / H, h = bh % H;
    const size_t o = at3(b, h, 0, H, T);
    decode_head<double>(T, din, dout, x + o * din, v + o * dout, eta + o, alpha + o,
                        W0 + (size_t)h * dd, S + (size_t)bh * dd, y + o * dout, g + o * dout);
  }
}

// Two-layer serial learner (see mlp2_serial_head): y, g1, g2 for every pair.
// x [B,H,T,dx], v/y/g2 [B,H,T,dy], g1 [B,H,T,dh], W1 [H,dh,dx], W2 [H,dy,dh].
void oracle_mlp2_serial_f64(int B, int H, int T, int dx, int dh, int dy, const double* x,
                            const double* v, const double* eta, const double* alpha,
                            const double* W1, const double* W2, double* y, double* g1,
                            double* g2, int nthreads) {
  const int nt = pick_threads(nthreads);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
    const int h = bh % H;
    const size_t o = (size_t)bh * T;
    mlp2_serial_head<double>(T, dx, dh, dy, x + o * dx, v + o * dy, eta + o, alpha + o,
                             W1 + (size_t)h * dh * dx, W2 + (size_t)h * dy * dh, y + o * dy,
                             g1 + o * dh, g2 + o * dy);
  }
}

// Two-layer parallel reconstruction (see mlp2_recon_head). a, h, g1til [B,H,T,dh];
// y, g2til [B,H,T,dy]; dW1 [B,H,dh,dx].
void oracle_mlp2_recon_f64(int B, int H, int T, int dx, int dh, int dy, const double* x,
                           const double* g1hat, const double* g2hat, const double* v,
                           const double* eta, const double* alpha, const double* W1,
                           const double* W2, int control, double* a, double* hh, double* y,
                           double* g2til, double* g1til, double* dW1, int nthreads) {
  const int nt = pick_threads(nthreads);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
    const int h = bh % H;
    const size_t o = (size_t)bh * T;
    mlp2_recon_head(T, dx, dh, dy, x + o * dx, g1hat + o * dh, g2hat + o * dy, v + o * dy,
                    eta + o, alpha + o, W1 + (size_t)h * dh * dx, W2 + (size_t)h * dy * dh,
                    control, a + o * dh, hh + o * dh, y + o * dy, g2til + o * dy,
                    g1til + o * dh, dW1 + (size_t)bh * dh * dx);
  }
}

int oracle_max_threads(void) { return pick_threads(0); }

}  // extern "C"
