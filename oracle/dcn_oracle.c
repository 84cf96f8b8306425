/*
 * CPU oracle for the DCNv3 / DCNv4 core operator.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The CUDA
 * library shares no code, header, table or helper with it.
 *
 * What is computed (InternImage-L DCNv3 explainer (wmrh.cn), section 二,
 * steps 2-4, and section 三): for every output pixel (n, ho, wo) and group g
 * the operator takes, for each of the K*K taps k = a*K + b, a learned offset
 * (dx, dy) scaled by offset_scale, samples the group's Cg input channels
 * bilinearly at the displaced grid point (zero outside the image), and sums
 * the samples weighted by a per-group mask.  For DCNv3 the mask holds
 * logits and is normalised with a softmax over the K*K taps of the group
 * (step 3); for the DCNv4 variant the mask is used as given.
 *
 *   out[n,ho,wo,g,c] = sum_k m[n,ho,wo,g,k] * B(x[n,:,:,g,c]; Y_k, X_k)
 *   Y_k = ho*s - p + a*d + sigma*dy_k,   X_k = wo*s - p + b*d + sigma*dx_k
 *   B(f; Y, X) = sum over the 4 corners (yc, xc) of floor(Y,X)+{0,1}^2 of
 *                wy(yc) * wx(xc) * f[yc, xc], corners outside the image are 0,
 *                wx(x0) = 1 - (X - x0), wx(x0 + 1) = X - x0 (same for y).
 *
 * Readings of points the pages leave open (each one is listed with its
 * reason in the design notes):
 *  - integer (Y, X) is a pixel centre: zero offsets reproduce the plain
 *    convolution grid, which is what the explainer's "starts out as a plain
 *    3x3 convolution" remark needs;
 *  - zero padding per corner; a sample contributes (and has a derivative)
 *    only when -1 <= Y < H and -1 <= X < W, which also drops NaN and inf;
 *  - the sampling grid is the usual convolution grid ho*s - p + a*d, with a
 *    stride, padding and dilation per axis (the height ones apply to ho and
 *    a, the width ones to wo and b; the pages' modules take one value for
 *    both, which is the case stride_w = stride and so on);
 *  - offsets are stored as (dx, dy) pairs, taps row-major (k = a*K + b);
 *  - the softmax subtracts the per-group maximum before exponentiating;
 *  - location rounding: in "fp32-location" mode (fd = 0) each of
 *    sigma*dy and base + (sigma*dy) is rounded to fp32 separately, as the
 *    CUDA path does, so both land in the same floor cell; in "fd" mode
 *    (fd = 1) everything is double, for finite differences;
 *  - the gradient at an integer coordinate is the one-sided derivative that
 *    floor() selects (corners x0 = X and X + 1);
 *  - remove_center (a DCNv4 module argument, DCNv4 speed-up write-up
 *    (pnsm.cn), section 3.3, which drops the centre sampling point): the taps
 *    are the K x K window positions in row-major order with the centre
 *    position (K/2, K/2) left out, so there are T = K*K - 1 of them and
 *    offset and mask carry T entries per group; without it T = K*K.
 *
 * All accumulation is in double.  Inputs are double arrays holding the exact
 * values of the fp32 / bf16 tensors the CUDA path sees.
 *
 * Layouts (element indices, C = G*Cg, T taps per group):
 *   x      ((n*H + y)*W + x)*C + g*Cg + c
 *   offset ((n*Ho + ho)*Wo + wo)*(G*T*2) + (g*T + k)*2 + {0: dx, 1: dy}
 *   mask   ((n*Ho + ho)*Wo + wo)*(G*T) + g*T + k
 *   out    ((n*Ho + ho)*Wo + wo)*C + g*Cg + c
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t N, H, W, G, Cg, K, Ho, Wo;
  int64_t stride, pad, dil;        /* height axis */
  int64_t stride_w, pad_w, dil_w;  /* width axis */
  int64_t T; /* taps per (pixel, group) */
  double sigma;
  int softmax, fd, remove_center;
} prob_t;

/* Output extent of a convolution grid; 0 when no tap window fits. */
int oracle_output_extent(int in, int K, int stride, int pad, int dil) {
  int64_t span = (int64_t)in + 2 * (int64_t)pad - (int64_t)dil * (K - 1) - 1;
  if (span < 0 || stride < 1) return 0;
  return (int)(span / stride + 1);
}

static prob_t make_prob(int N, int H, int W, int G, int Cg, int K, int stride,
                        int pad, int dil, double sigma, int softmax, int fd,
                        int remove_center, int stride_w, int pad_w, int dil_w) {
  prob_t p;
  p.N = N; p.H = H; p.W = W; p.G = G; p.Cg = Cg; p.K = K;
  p.stride = stride; p.pad = pad; p.dil = dil;
  p.stride_w = stride_w; p.pad_w = pad_w; p.dil_w = dil_w;
  p.Ho = oracle_output_extent(H, K, stride, pad, dil);
  p.Wo = oracle_output_extent(W, K, stride_w, pad_w, dil_w);
  p.sigma = sigma; p.softmax = softmax; p.fd = fd;
  p.remove_center = remove_center != 0;
  p.T = (int64_t)K * K - p.remove_center;
  return p;
}

/* A problem the oracle can evaluate: a non-empty output and at least one tap. */
static int usable(const prob_t* p) { return p->Ho > 0 && p->Wo > 0 && p->T > 0; }

/* Window position (a, b) of tap j: the K x K positions are listed row by
 * row, skipping the centre when remove_center is set, and tap j is the j-th
 * entry of that list. */
static void tap_position(const prob_t* p, int64_t j, int64_t* a, int64_t* b) {
  int64_t listed = 0;
  *a = *b = 0;
  for (int64_t r = 0; r < p->K; ++r) {
    for (int64_t c = 0; c < p->K; ++c) {
      if (p->remove_center && r == p->K / 2 && c == p->K / 2) continue;
      if (listed == j) {
        *a = r;
        *b = c;
        return;
      }
      ++listed;
    }
  }
}

/* Mask weights of one (pixel, group): softmax over its KK taps (DCNv3,
 * explainer section 二 step 3) or the raw values (DCNv4). */
static void mask_weights(const double* logits, int64_t KK, int softmax, double* m) {
  if (!softmax) {
    for (int64_t k = 0; k < KK; ++k) m[k] = logits[k];
    return;
  }
  double mx = logits[0];
  for (int64_t k = 1; k < KK; ++k) if (logits[k] > mx) mx = logits[k];
  double sum = 0.0;
  for (int64_t k = 0; k < KK; ++k) { m[k] = exp(logits[k] - mx); sum += m[k]; }
  for (int64_t k = 0; k < KK; ++k) m[k] /= sum;
}

/* Sampling location of tap (a, b) of output pixel (ho, wo). */
static void location(const prob_t* p, int64_t ho, int64_t wo, int64_t a, int64_t b,
                     double dx, double dy, double* Y, double* X) {
  int64_t base_y = ho * p->stride - p->pad + a * p->dil;
  int64_t base_x = wo * p->stride_w - p->pad_w + b * p->dil_w;
  if (p->fd) {
    *Y = (double)base_y + p->sigma * dy;
    *X = (double)base_x + p->sigma * dx;
  } else {
    /* Two separately rounded fp32 operations (no fused multiply-add: the
     * library is built with -ffp-contract=off). */
    float s = (float)p->sigma;
    float ty = s * (float)dy;
    float tx = s * (float)dx;
    float yf = (float)base_y + ty;
    float xf = (float)base_x + tx;
    *Y = (double)yf;
    *X = (double)xf;
  }
}

static int in_support(const prob_t* p, double Y, double X) {
  return Y >= -1.0 && Y < (double)p->H && X >= -1.0 && X < (double)p->W;
}

static const double* pixel_ptr(const prob_t* p, const double* t, int64_t n,
                               int64_t y, int64_t x, int64_t g) {
  return t + ((n * p->H + y) * p->W + x) * (p->G * p->Cg) + g * p->Cg;
}

/* Forward of one unit (n, ho, wo, g): writes Cg outputs to out_c. */
static void forward_unit(const prob_t* p, const double* x, const double* off,
                         const double* mask, int64_t n, int64_t ho, int64_t wo,
                         int64_t g, double* out_c) {
  const int64_t KK = p->T;
  const int64_t pix = (n * p->Ho + ho) * p->Wo + wo;
  const double* o = off + pix * (p->G * KK * 2) + g * KK * 2;
  const double* l = mask + pix * (p->G * KK) + g * KK;
  double* m = (double*)malloc(sizeof(double) * (size_t)KK);
  mask_weights(l, KK, p->softmax, m);
  for (int64_t c = 0; c < p->Cg; ++c) out_c[c] = 0.0;
  for (int64_t k = 0; k < KK; ++k) {
    int64_t a, b;
    tap_position(p, k, &a, &b);
    double Y, X;
    location(p, ho, wo, a, b, o[2 * k], o[2 * k + 1], &Y, &X);
    if (!in_support(p, Y, X)) continue;
    const double y0 = floor(Y), x0 = floor(X);
    const double ly = Y - y0, lx = X - x0;
    for (int cy = 0; cy < 2; ++cy) {
      for (int cx = 0; cx < 2; ++cx) {
        const int64_t yc = (int64_t)y0 + cy, xc = (int64_t)x0 + cx;
        if (yc < 0 || yc >= p->H || xc < 0 || xc >= p->W) continue;
        const double wy = cy ? ly : 1.0 - ly;
        const double wx = cx ? lx : 1.0 - lx;
        const double* f = pixel_ptr(p, x, n, yc, xc, g);
        for (int64_t c = 0; c < p->Cg; ++c) out_c[c] += m[k] * (wy * wx * f[c]);
      }
    }
  }
  free(m);
}

/*
 * Full forward.  x: (N,H,W,G*Cg); offset: (N,Ho,Wo,G*T*2); mask: (N,Ho,Wo,G*T)
 * with T = K*K - remove_center; out: (N,Ho,Wo,G*Cg).  Returns 0, or -1 when
 * the output would be empty or there is no tap.
 */
int oracle_forward(const double* x, const double* offset, const double* mask,
                   double* out, int N, int H, int W, int G, int Cg, int K,
                   int stride, int pad, int dil, double sigma, int softmax, int fd,
                   int remove_center, int stride_w, int pad_w, int dil_w) {
  prob_t p = make_prob(N, H, W, G, Cg, K, stride, pad, dil, sigma, softmax, fd, remove_center,
                       stride_w, pad_w, dil_w);
  if (!usable(&p)) return -1;
  for (int64_t n = 0; n < p.N; ++n)
    for (int64_t ho = 0; ho < p.Ho; ++ho)
      for (int64_t wo = 0; wo < p.Wo; ++wo)
        for (int64_t g = 0; g < p.G; ++g)
          forward_unit(&p, x, offset, mask, n, ho, wo, g,
                       out + ((n * p.Ho + ho) * p.Wo + wo) * (p.G * p.Cg) + g * p.Cg);
  return 0;
}

/*
 * Forward of selected units only: unit u = ((n*Ho + ho)*Wo + wo)*G + g.
 * out: (n_units, Cg).  For checking large problems on sampled outputs.
 */
int oracle_forward_units(const double* x, const double* offset, const double* mask,
                         const int64_t* units, int64_t n_units, double* out, int N,
                         int H, int W, int G, int Cg, int K, int stride, int pad,
                         int dil, double sigma, int softmax, int fd, int remove_center,
                         int stride_w, int pad_w, int dil_w) {
  prob_t p = make_prob(N, H, W, G, Cg, K, stride, pad, dil, sigma, softmax, fd, remove_center,
                       stride_w, pad_w, dil_w);
  if (!usable(&p)) return -1;
  for (int64_t i = 0; i < n_units; ++i) {
    int64_t u = units[i];
    int64_t g = u % p.G, pix = u / p.G;
    int64_t wo = pix % p.Wo, t = pix / p.Wo;
    int64_t ho = t % p.Ho, n = t / p.Ho;
    if (n >= p.N || u < 0) return -2;
    forward_unit(&p, x, offset, mask, n, ho, wo, g, out + i * p.Cg);
  }
  return 0;
}

/*
 * Backward of one unit.  Writes the unit's offset and mask gradients
 * (goff: T*2 values, gmask: T values) and, when gx != NULL, adds the
 * unit's contribution to the input gradient.
 *
 *   v_k[c]   = B(x[.,.,g,c]; Y_k, X_k)                      (unweighted sample)
 *   s_k      = sum_c gout[c] * v_k[c]
 *   dv/dX[c] = sum_yc wy(yc) * (f[yc, x0+1] - f[yc, x0])    (out-of-image corners 0)
 *   dv/dY[c] = sum_xc wx(xc) * (f[y0+1, xc] - f[y0, xc])
 *   goff[k]  = sigma * m_k * sum_c gout[c] * (dv/dX[c], dv/dY[c])
 *   softmax:  glogit_k = m_k * (s_k - sum_j m_j s_j);  else gmask_k = s_k
 *   gx[corner, c] += m_k * wy * wx * gout[c]
 */
static void backward_unit(const prob_t* p, const double* x, const double* off,
                          const double* mask, const double* gout, int64_t n,
                          int64_t ho, int64_t wo, int64_t g, double* gx,
                          double* goff_u, double* gmask_u) {
  const int64_t KK = p->T, C = p->G * p->Cg;
  const int64_t pix = (n * p->Ho + ho) * p->Wo + wo;
  const double* o = off + pix * (p->G * KK * 2) + g * KK * 2;
  const double* l = mask + pix * (p->G * KK) + g * KK;
  const double* go = gout + pix * C + g * p->Cg;
  double* m = (double*)malloc(sizeof(double) * (size_t)KK);
  double* s = (double*)malloc(sizeof(double) * (size_t)KK);
  mask_weights(l, KK, p->softmax, m);
  for (int64_t k = 0; k < KK; ++k) {
    int64_t a, b;
    tap_position(p, k, &a, &b);
    double Y, X;
    location(p, ho, wo, a, b, o[2 * k], o[2 * k + 1], &Y, &X);
    s[k] = 0.0;
    goff_u[2 * k] = 0.0;
    goff_u[2 * k + 1] = 0.0;
    if (!in_support(p, Y, X)) continue;
    const int64_t y0 = (int64_t)floor(Y), x0 = (int64_t)floor(X);
    const double ly = Y - (double)y0, lx = X - (double)x0;
    double gX = 0.0, gY = 0.0;
    for (int cy = 0; cy < 2; ++cy) {
      for (int cx = 0; cx < 2; ++cx) {
        const int64_t yc = y0 + cy, xc = x0 + cx;
        if (yc < 0 || yc >= p->H || xc < 0 || xc >= p->W) continue;
        const double wy = cy ? ly : 1.0 - ly;
        const double wx = cx ? lx : 1.0 - lx;
        const double dwx = cx ? 1.0 : -1.0; /* d wx / dX */
        const double dwy = cy ? 1.0 : -1.0; /* d wy / dY */
        const double* f = pixel_ptr(p, x, n, yc, xc, g);
        for (int64_t c = 0; c < p->Cg; ++c) {
          s[k] += go[c] * (wy * wx * f[c]);
          gX += go[c] * (wy * dwx * f[c]);
          gY += go[c] * (dwy * wx * f[c]);
        }
        if (gx) {
          double* gf = gx + ((n * p->H + yc) * p->W + xc) * C + g * p->Cg;
          for (int64_t c = 0; c < p->Cg; ++c) gf[c] += m[k] * wy * wx * go[c];
        }
      }
    }
    goff_u[2 * k] = p->sigma * m[k] * gX;
    goff_u[2 * k + 1] = p->sigma * m[k] * gY;
  }
  if (p->softmax) {
    double ms = 0.0;
    for (int64_t k = 0; k < KK; ++k) ms += m[k] * s[k];
    for (int64_t k = 0; k < KK; ++k) gmask_u[k] = m[k] * (s[k] - ms);
  } else {
    for (int64_t k = 0; k < KK; ++k) gmask_u[k] = s[k];
  }
  free(m);
  free(s);
}

/*
 * Full backward.  grad_input is overwritten (zero-filled, then accumulated);
 * grad_offset and grad_mask are overwritten.  With softmax, grad_mask is the
 * gradient with respect to the logits.
 */
int oracle_backward(const double* x, const double* offset, const double* mask,
                    const double* grad_out, double* grad_input, double* grad_offset,
                    double* grad_mask, int N, int H, int W, int G, int Cg, int K,
                    int stride, int pad, int dil, double sigma, int softmax, int fd,
                    int remove_center, int stride_w, int pad_w, int dil_w) {
  prob_t p = make_prob(N, H, W, G, Cg, K, stride, pad, dil, sigma, softmax, fd, remove_center,
                       stride_w, pad_w, dil_w);
  if (!usable(&p)) return -1;
  const int64_t KK = p.T;
  memset(grad_input, 0, sizeof(double) * (size_t)(p.N * p.H * p.W * p.G * p.Cg));
  for (int64_t n = 0; n < p.N; ++n)
    for (int64_t ho = 0; ho < p.Ho; ++ho)
      for (int64_t wo = 0; wo < p.Wo; ++wo)
        for (int64_t g = 0; g < p.G; ++g) {
          const int64_t u = ((n * p.Ho + ho) * p.Wo + wo) * p.G + g;
          backward_unit(&p, x, offset, mask, grad_out, n, ho, wo, g, grad_input,
                        grad_offset + u * KK * 2, grad_mask + u * KK);
        }
  return 0;
}

/* Offset and mask gradients of selected units (no input gradient).
 * goff: (n_units, T*2), gmask: (n_units, T). */
int oracle_backward_units(const double* x, const double* offset, const double* mask,
                          const double* grad_out, const int64_t* units, int64_t n_units,
                          double* goff, double* gmask, int N, int H, int W, int G,
                          int Cg, int K, int stride, int pad, int dil, double sigma,
                          int softmax, int fd, int remove_center, int stride_w, int pad_w,
                          int dil_w) {
  prob_t p = make_prob(N, H, W, G, Cg, K, stride, pad, dil, sigma, softmax, fd, remove_center,
                       stride_w, pad_w, dil_w);
  if (!usable(&p)) return -1;
  const int64_t KK = p.T;
  for (int64_t i = 0; i < n_units; ++i) {
    int64_t u = units[i];
    int64_t g = u % p.G, pix = u / p.G;
    int64_t wo = pix % p.Wo, t = pix / p.Wo;
    int64_t ho = t % p.Ho, n = t / p.Ho;
    if (n >= p.N || u < 0) return -2;
    backward_unit(&p, x, offset, mask, grad_out, n, ho, wo, g, NULL,
                  goff + i * KK * 2, gmask + i * KK);
  }
  return 0;
}
