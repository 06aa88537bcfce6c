/*
 * Plain CPU oracle for the per-sample kernel-mixture convolution.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library. The product path (the CUDA C-ABI
 * library) never calls it and shares no code, header, table or helper with it.
 *
 * Everything here is fp64, written as the definition reads, with direct nested
 * loops and no blocking, fusion or reordering. Threads split the work over
 * samples only; each sample is computed exactly as a single thread would.
 *
 * What is computed, and where it comes from:
 *   routing   alpha_b = act(FC(GAP(x_b)))  -- attentions computed from the
 *             input (KernelWarehouse: Rethinking the Design of Dynamic Convolution,
 *             abstract), one attention vector per example (CondConv:
 *             Conditionally Parameterized Convolutions for Efficient Inference,
 *             abstract); the temperature divides the logits before the softmax
 *             (the kernel attention carries a temperature, FMDConv: Fast
 *             multi-attention dynamic convolution via speed-accuracy trade-off,
 *             abstract). The GAP -> single linear layer -> sigmoid/softmax form
 *             is the reading taken where the pages are silent.
 *   assembly  W_b = sum_i alpha_{b,i} W_i, b_b = sum_i alpha_{b,i} bias_i
 *             (n static kernels summed with weights that depend on the
 *             input, KernelWarehouse abstract).
 *   conv      y_b = conv2d(x_b, W_b) + b_b, cross-correlation with zero padding
 *             (a kernel specialised to each example, CondConv abstract);
 *             orientation and padding are readings, pinned by tests.
 *
 * Layouts (all row-major, fastest index last):
 *   x       [B][H][W][C_in]                      (NHWC)
 *   experts [n][C_out][KH][KW][C_in/groups]
 *   Wr      [n][C_in],  br [n]
 *   bias    [n][C_out]  (may be NULL: no bias)
 *   alpha   [B][n]
 *   y       [B][H_out][W_out][C_out]             (NHWC)
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_SIGMOID 0
#define ORACLE_SOFTMAX 1

/* ---------------------------------------------------------------- threads */

typedef void (*sample_fn)(void *ctx, int b);

typedef struct {
  sample_fn fn;
  void *ctx;
  int next;           /* next sample to take */
  int end;
  pthread_mutex_t mu;
} pool_t;

static void *pool_worker(void *arg) {
  pool_t *p = (pool_t *)arg;
  for (;;) {
    pthread_mutex_lock(&p->mu);
    int b = p->next < p->end ? p->next++ : -1;
    pthread_mutex_unlock(&p->mu);
    if (b < 0) return NULL;
    p->fn(p->ctx, b);
  }
}

static int run_samples(sample_fn fn, void *ctx, int b0, int nb, int nthreads) {
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nb) nthreads = nb;
  pool_t p;
  p.fn = fn; p.ctx = ctx; p.next = b0; p.end = b0 + nb;
  pthread_mutex_init(&p.mu, NULL);
  if (nthreads <= 1) {
    pool_worker(&p);
  } else {
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -1;
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, pool_worker, &p);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
  }
  pthread_mutex_destroy(&p.mu);
  return 0;
}

int oracle_threads_used(int nthreads, int nb) {
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nb) nthreads = nb;
  return nthreads;
}

/* ---------------------------------------------------------------- routing */

/* Step 1: g[c] = (1/(H*W)) * sum over the H*W unpadded pixels of x[b,h,w,c]. */
void oracle_gap(int C, int H, int W, const double *xb, double *g) {
  for (int c = 0; c < C; ++c) {
    double s = 0.0;
    for (int h = 0; h < H; ++h)
      for (int w = 0; w < W; ++w)
        s += xb[((size_t)h * W + w) * C + c];
    g[c] = s / (double)(H * W);
  }
}

/* Step 2: z[i] = br[i] + sum_c Wr[i,c] * g[c]   (one linear layer). */
void oracle_fc(int C, int n, const double *Wr, const double *br, const double *g, double *z) {
  for (int i = 0; i < n; ++i) {
    double s = br ? br[i] : 0.0;
    for (int c = 0; c < C; ++c) s += Wr[(size_t)i * C + c] * g[c];
    z[i] = s;
  }
}

/* Step 3: sigmoid per expert, or softmax over experts of z/tau.
 * Written without max-subtraction: in fp64 the logits here never overflow. */
void oracle_act(int n, const double *z, int mode, double tau, double *alpha) {
  if (mode == ORACLE_SIGMOID) {
    for (int i = 0; i < n; ++i) alpha[i] = 1.0 / (1.0 + exp(-z[i]));
  } else {
    double den = 0.0;
    for (int j = 0; j < n; ++j) den += exp(z[j] / tau);
    for (int i = 0; i < n; ++i) alpha[i] = exp(z[i] / tau) / den;
  }
}

typedef struct {
  int C, H, W, n, mode;
  double tau;
  const double *x, *Wr, *br;
  double *alpha;
} route_ctx;

static void route_one(void *vctx, int b) {
  route_ctx *r = (route_ctx *)vctx;
  double *g = (double *)malloc(sizeof(double) * (size_t)r->C);
  double *z = (double *)malloc(sizeof(double) * (size_t)r->n);
  const double *xb = r->x + (size_t)b * r->H * r->W * r->C;
  oracle_gap(r->C, r->H, r->W, xb, g);
  oracle_fc(r->C, r->n, r->Wr, r->br, g, z);
  oracle_act(r->n, z, r->mode, r->tau, r->alpha + (size_t)b * r->n);
  free(g);
  free(z);
}

/* alpha[B][n] for every sample. Returns 0, or -1 on a bad argument. */
int oracle_route(int B, int C, int H, int W, const double *x, int n, const double *Wr,
                 const double *br, int mode, double tau, double *alpha, int nthreads) {
  if (B < 0 || C <= 0 || H <= 0 || W <= 0 || n <= 0 || !x || !Wr || !alpha) return -1;
  if (mode != ORACLE_SIGMOID && mode != ORACLE_SOFTMAX) return -1;
  if (mode == ORACLE_SOFTMAX && !(tau > 0.0)) return -1;
  if (B == 0) return 0;
  route_ctx r = {C, H, W, n, mode, tau, x, Wr, br, alpha};
  return run_samples(route_one, &r, 0, B, nthreads);
}

/* ---------------------------------------------------------- assembly + conv */

/* Step 4: W_b = sum_i alpha_i W_i over every weight element, and the mixed bias. */
void oracle_assemble(int n, long wsize, const double *experts, const double *alpha_b,
                     double *Wb) {
  for (long e = 0; e < wsize; ++e) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += alpha_b[i] * experts[(size_t)i * wsize + e];
    Wb[e] = s;
  }
}

void oracle_mix_bias(int n, int Cout, const double *bias, const double *alpha_b, double *bb) {
  for (int co = 0; co < Cout; ++co) {
    double s = 0.0;
    if (bias)
      for (int i = 0; i < n; ++i) s += alpha_b[i] * bias[(size_t)i * Cout + co];
    bb[co] = s;
  }
}

typedef struct {
  int Cin, H, W, Cout, KH, KW, stride, pad, groups, n, Ho, Wo, b0;
  int oh_begin, oh_end;   /* output rows computed, [oh_begin, oh_end) */
  const double *x, *experts, *alpha, *bias;
  double *y;              /* rows oh_begin.. of samples b0.. */
  const double *a_in;     /* [B][Cin] input (channel) attention, or NULL: all ones */
  const double *a_out;    /* [B][Cout] output (channel) attention, or NULL: all ones */
} fwd_ctx;

static void forward_one(void *vctx, int b) {
  fwd_ctx *f = (fwd_ctx *)vctx;
  const int Cg = f->Cin / f->groups;       /* input channels seen by one output channel */
  const int Coutg = f->Cout / f->groups;   /* output channels per group */
  const long wsize = (long)f->Cout * f->KH * f->KW * Cg;
  double *Wb = (double *)malloc(sizeof(double) * (size_t)wsize);
  double *bb = (double *)malloc(sizeof(double) * (size_t)f->Cout);
  const double *ab = f->alpha + (size_t)b * f->n;
  oracle_assemble(f->n, wsize, f->experts, ab, Wb);
  oracle_mix_bias(f->n, f->Cout, f->bias, ab, bb);

  /* Step 5: y[oh,ow,co] = b_b[co] + sum_{kh,kw,ci} xpad[oh*s+kh-p, ow*s+kw-p, g*Cg+ci] W_b[co,kh,kw,ci]
   * With the FMDConv channel attentions (FMDConv, abstract: input attention and
   * output attention; no formula on the page, reading: per-channel factors of
   * the sample): the input factor multiplies x channel by channel, the output
   * factor multiplies y (bias included) channel by channel. */
  const double *xb = f->x + (size_t)b * f->H * f->W * f->Cin;
  const double *ain = f->a_in ? f->a_in + (size_t)b * f->Cin : NULL;
  const double *aout = f->a_out ? f->a_out + (size_t)b * f->Cout : NULL;
  const int nrows = f->oh_end - f->oh_begin;
  double *yb = f->y + (size_t)(b - f->b0) * nrows * f->Wo * f->Cout;
  for (int oh = f->oh_begin; oh < f->oh_end; ++oh)
    for (int ow = 0; ow < f->Wo; ++ow)
      for (int co = 0; co < f->Cout; ++co) {
        const int g = co / Coutg;
        double s = bb[co];
        for (int kh = 0; kh < f->KH; ++kh) {
          const int ih = oh * f->stride + kh - f->pad;
          if (ih < 0 || ih >= f->H) continue;          /* zero padding */
          for (int kw = 0; kw < f->KW; ++kw) {
            const int iw = ow * f->stride + kw - f->pad;
            if (iw < 0 || iw >= f->W) continue;        /* zero padding */
            const double *xp = xb + ((size_t)ih * f->W + iw) * f->Cin + (size_t)g * Cg;
            const double *wp = Wb + (((size_t)co * f->KH + kh) * f->KW + kw) * Cg;
            if (ain) {
              const double *ap = ain + (size_t)g * Cg;
              for (int ci = 0; ci < Cg; ++ci) s += (ap[ci] * xp[ci]) * wp[ci];
            } else {
              for (int ci = 0; ci < Cg; ++ci) s += xp[ci] * wp[ci];
            }
          }
        }
        if (aout) s *= aout[co];
        yb[((size_t)(oh - f->oh_begin) * f->Wo + ow) * f->Cout + co] = s;
      }
  free(Wb);
  free(bb);
}

int oracle_out_size(int in, int k, int stride, int pad) {
  return (in + 2 * pad - k) / stride + 1;
}

/* y for samples b0 .. b0+nb-1, written to y[nb][Ho][Wo][Cout].
 * Returns 0, or -1 on a bad argument. */
int oracle_forward(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride, int pad,
                   int groups, int n, const double *x, const double *experts,
                   const double *alpha, const double *bias, int b0, int nb, double *y,
                   int nthreads) {
  if (B < 0 || Cin <= 0 || H <= 0 || W <= 0 || Cout <= 0 || KH <= 0 || KW <= 0) return -1;
  if (stride <= 0 || pad < 0 || groups <= 0 || n <= 0) return -1;
  if (Cin % groups != 0 || Cout % groups != 0) return -1;
  if (!x || !experts || !alpha || !y) return -1;
  if (b0 < 0 || nb < 0 || b0 + nb > B) return -1;
  const int Ho = oracle_out_size(H, KH, stride, pad), Wo = oracle_out_size(W, KW, stride, pad);
  if (Ho <= 0 || Wo <= 0) return -1;
  if (nb == 0) return 0;
  fwd_ctx f = {Cin, H, W, Cout, KH, KW, stride, pad, groups, n, Ho, Wo, b0, 0, Ho,
               x, experts, alpha, bias, y, NULL, NULL};
  return run_samples(forward_one, &f, b0, nb, nthreads);
}

/* oracle_forward with the FMDConv channel attentions: a_in [B][Cin] multiplies
 * the input channels of each sample, a_out [B][Cout] its output channels (bias
 * included); either may be NULL (all ones). */
int oracle_forward_attn(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                        int pad, int groups, int n, const double *x, const double *experts,
                        const double *alpha, const double *bias, const double *a_in,
                        const double *a_out, int b0, int nb, double *y, int nthreads) {
  if (B < 0 || Cin <= 0 || H <= 0 || W <= 0 || Cout <= 0 || KH <= 0 || KW <= 0) return -1;
  if (stride <= 0 || pad < 0 || groups <= 0 || n <= 0) return -1;
  if (Cin % groups != 0 || Cout % groups != 0) return -1;
  if (!x || !experts || !alpha || !y) return -1;
  if (b0 < 0 || nb < 0 || b0 + nb > B) return -1;
  const int Ho = oracle_out_size(H, KH, stride, pad), Wo = oracle_out_size(W, KW, stride, pad);
  if (Ho <= 0 || Wo <= 0) return -1;
  if (nb == 0) return 0;
  fwd_ctx f = {Cin, H, W, Cout, KH, KW, stride, pad, groups, n, Ho, Wo, b0, 0, Ho,
               x, experts, alpha, bias, y, a_in, a_out};
  return run_samples(forward_one, &f, b0, nb, nthreads);
}

/* Output rows oh0 .. oh0+noh-1 of sample b only, written to y[noh][Wo][Cout]
 * (the same definition restricted to a band of output rows; single thread). */
int oracle_forward_rows(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                        int pad, int groups, int n, const double *x, const double *experts,
                        const double *alpha, const double *bias, int b, int oh0, int noh,
                        double *y) {
  if (B <= 0 || Cin <= 0 || H <= 0 || W <= 0 || Cout <= 0 || KH <= 0 || KW <= 0) return -1;
  if (stride <= 0 || pad < 0 || groups <= 0 || n <= 0) return -1;
  if (Cin % groups != 0 || Cout % groups != 0) return -1;
  if (!x || !experts || !alpha || !y) return -1;
  const int Ho = oracle_out_size(H, KH, stride, pad), Wo = oracle_out_size(W, KW, stride, pad);
  if (Ho <= 0 || Wo <= 0 || b < 0 || b >= B || oh0 < 0 || noh < 0 || oh0 + noh > Ho) return -1;
  if (noh == 0) return 0;
  fwd_ctx f = {Cin, H, W, Cout, KH, KW, stride, pad, groups, n, Ho, Wo, b, oh0, oh0 + noh,
               x, experts, alpha, bias, y, NULL, NULL};
  forward_one(&f, b);
  return 0;
}

/* =============================================================== backward */
/*
 * Gradients of a scalar loss through one layer, given dy = dL/dy
 * [B][Ho][Wo][Cout]. The per-example kernels and the mixture are learned
 * (CondConv, abstract; KernelWarehouse, abstract), so the layer is trained
 * through the derivative of the definition above. Each function is that
 * derivative, one forward step at a time (chain rule), written as plainly as
 * the forward:
 *
 *   conv      dW_b[co,kh,kw,ci] = sum_{oh,ow} dy[b,oh,ow,co] xpad[b, oh*s+kh-p, ow*s+kw-p, g*Cg+ci]
 *             db_b[co]          = sum_{oh,ow} dy[b,oh,ow,co]
 *             dx_b              = every dy[b,oh,ow,co] * W_b[co,kh,kw,ci] added back onto the
 *                                 input element that the forward read with it
 *   assembly  dexperts_i = sum_b alpha[b,i] dW_b        dbias_i = sum_b alpha[b,i] db_b
 *             dalpha[b,i] = <dW_b, W_i> + <db_b, bias_i>
 *   act       sigmoid: dz = dalpha * alpha * (1 - alpha)
 *             softmax of z/tau: dz_i = alpha_i * (dalpha_i - sum_j alpha_j dalpha_j) / tau
 *   FC        dWr[i,c] = sum_b dz[b,i] g[b,c],  dbr[i] = sum_b dz[b,i],
 *             dg[b,c] = sum_i dz[b,i] Wr[i,c]
 *   GAP       dx[b,h,w,c] += dg[b,c] / (H*W)   (every unpadded pixel)
 */

typedef struct {
  int Cin, H, W, Cout, KH, KW, stride, pad, groups, Ho, Wo, b0;
  const double *x, *dy;
  double *dW;   /* [nb][Cout][KH][KW][Cg] */
  double *db;   /* [nb][Cout] */
} wgrad_ctx;

static void wgrad_one(void *vctx, int b) {
  wgrad_ctx *f = (wgrad_ctx *)vctx;
  const int Cg = f->Cin / f->groups, Coutg = f->Cout / f->groups;
  const long wsize = (long)f->Cout * f->KH * f->KW * Cg;
  double *dW = f->dW + (size_t)(b - f->b0) * wsize;
  double *db = f->db + (size_t)(b - f->b0) * f->Cout;
  memset(dW, 0, sizeof(double) * (size_t)wsize);
  memset(db, 0, sizeof(double) * (size_t)f->Cout);
  const double *xb = f->x + (size_t)b * f->H * f->W * f->Cin;
  const double *dyb = f->dy + (size_t)b * f->Ho * f->Wo * f->Cout;
  for (int oh = 0; oh < f->Ho; ++oh)
    for (int ow = 0; ow < f->Wo; ++ow)
      for (int co = 0; co < f->Cout; ++co) {
        const double d = dyb[((size_t)oh * f->Wo + ow) * f->Cout + co];
        const size_t cin0 = (size_t)(co / Coutg) * Cg;   /* first input channel of co's group */
        db[co] += d;
        for (int kh = 0; kh < f->KH; ++kh)
          for (int kw = 0; kw < f->KW; ++kw) {
            /* the input element the forward multiplied with W_b[co,kh,kw,.] */
            const int y_in = f->stride * oh - f->pad + kh, x_in = f->stride * ow - f->pad + kw;
            if (y_in < 0 || y_in >= f->H || x_in < 0 || x_in >= f->W) continue;  /* padding */
            const double *xp = xb + ((size_t)y_in * f->W + x_in) * f->Cin + cin0;
            double *gw = dW + ((size_t)(co * f->KH + kh) * f->KW + kw) * Cg;
            for (int ci = 0; ci < Cg; ++ci) gw[ci] += d * xp[ci];
          }
      }
}

static int bwd_shape_ok(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                        int pad, int groups, int n) {
  if (B < 0 || Cin <= 0 || H <= 0 || W <= 0 || Cout <= 0 || KH <= 0 || KW <= 0) return 0;
  if (stride <= 0 || pad < 0 || groups <= 0 || n <= 0) return 0;
  if (Cin % groups != 0 || Cout % groups != 0) return 0;
  if (oracle_out_size(H, KH, stride, pad) <= 0 || oracle_out_size(W, KW, stride, pad) <= 0)
    return 0;
  return 1;
}

/* Per-sample gradients of the convolution's weight and bias for samples
 * b0 .. b0+nb-1: dW[nb][Cout][KH][KW][Cin/groups], db[nb][Cout]. */
int oracle_weight_grad(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                       int pad, int groups, const double *x, const double *dy, int b0, int nb,
                       double *dW, double *db, int nthreads) {
  if (!bwd_shape_ok(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, 1)) return -1;
  if (!x || !dy || !dW || !db || b0 < 0 || nb < 0 || b0 + nb > B) return -1;
  if (nb == 0) return 0;
  wgrad_ctx f = {Cin, H, W, Cout, KH, KW, stride, pad, groups,
                 oracle_out_size(H, KH, stride, pad), oracle_out_size(W, KW, stride, pad), b0,
                 x, dy, dW, db};
  return run_samples(wgrad_one, &f, b0, nb, nthreads);
}

/* The assembly step's gradients: dexperts[n][wsize], dbias[n][Cout] (only when
 * bias is given) and dalpha[B][n], from the per-sample gradients of all B
 * samples. Sums over samples run in sample order. */
int oracle_backward_weight(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                           int pad, int groups, int n, const double *x, const double *dy,
                           const double *experts, const double *alpha, const double *bias,
                           double *dexperts, double *dbias, double *dalpha, int nthreads) {
  if (!bwd_shape_ok(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n)) return -1;
  if (!x || !dy || !experts || !alpha || !dexperts || !dalpha || (bias && !dbias)) return -1;
  const long wsize = (long)Cout * KH * KW * (Cin / groups);
  double *dW = (double *)malloc(sizeof(double) * (size_t)(B > 0 ? B : 1) * (size_t)wsize);
  double *db = (double *)malloc(sizeof(double) * (size_t)(B > 0 ? B : 1) * (size_t)Cout);
  if (!dW || !db) { free(dW); free(db); return -1; }
  int rc = B > 0 ? oracle_weight_grad(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, x, dy, 0,
                                      B, dW, db, nthreads)
                 : 0;
  if (rc == 0) {
    for (int b = 0; b < B; ++b)
      for (int i = 0; i < n; ++i) {
        double s = 0.0;
        for (long e = 0; e < wsize; ++e) s += dW[(size_t)b * wsize + e] * experts[(size_t)i * wsize + e];
        if (bias)
          for (int co = 0; co < Cout; ++co) s += db[(size_t)b * Cout + co] * bias[(size_t)i * Cout + co];
        dalpha[(size_t)b * n + i] = s;
      }
    for (int i = 0; i < n; ++i) {
      for (long e = 0; e < wsize; ++e) {
        double s = 0.0;
        for (int b = 0; b < B; ++b) s += alpha[(size_t)b * n + i] * dW[(size_t)b * wsize + e];
        dexperts[(size_t)i * wsize + e] = s;
      }
      if (bias)
        for (int co = 0; co < Cout; ++co) {
          double s = 0.0;
          for (int b = 0; b < B; ++b) s += alpha[(size_t)b * n + i] * db[(size_t)b * Cout + co];
          dbias[(size_t)i * Cout + co] = s;
        }
    }
  }
  free(dW);
  free(db);
  return rc;
}

/* The router's gradients: dz from dalpha through the activation, then the
 * linear layer's dWr[n][C], dbr[n] (sums over samples, in sample order) and
 * dg[B][C], the gradient of the pooled vector g of every sample. */
int oracle_route_backward(int B, int C, int H, int W, const double *x, int n, const double *Wr,
                          const double *alpha, const double *dalpha, int mode, double tau,
                          double *dWr, double *dbr, double *dg) {
  if (B < 0 || C <= 0 || H <= 0 || W <= 0 || n <= 0) return -1;
  if (!x || !Wr || !alpha || !dalpha || !dWr || !dbr || !dg) return -1;
  if (mode != ORACLE_SIGMOID && mode != ORACLE_SOFTMAX) return -1;
  if (mode == ORACLE_SOFTMAX && !(tau > 0.0)) return -1;
  double *g = (double *)malloc(sizeof(double) * (size_t)C);
  double *dz = (double *)malloc(sizeof(double) * (size_t)n);
  if (!g || !dz) { free(g); free(dz); return -1; }
  memset(dWr, 0, sizeof(double) * (size_t)n * C);
  memset(dbr, 0, sizeof(double) * (size_t)n);
  for (int b = 0; b < B; ++b) {
    const double *a = alpha + (size_t)b * n, *da = dalpha + (size_t)b * n;
    if (mode == ORACLE_SIGMOID) {
      for (int i = 0; i < n; ++i) dz[i] = da[i] * a[i] * (1.0 - a[i]);
    } else {
      double dot = 0.0;
      for (int j = 0; j < n; ++j) dot += a[j] * da[j];
      for (int i = 0; i < n; ++i) dz[i] = a[i] * (da[i] - dot) / tau;
    }
    oracle_gap(C, H, W, x + (size_t)b * H * W * C, g);
    for (int c = 0; c < C; ++c) {
      double s = 0.0;
      for (int i = 0; i < n; ++i) s += dz[i] * Wr[(size_t)i * C + c];
      dg[(size_t)b * C + c] = s;
    }
    for (int i = 0; i < n; ++i) {
      dbr[i] += dz[i];
      for (int c = 0; c < C; ++c) dWr[(size_t)i * C + c] += dz[i] * g[c];
    }
  }
  free(g);
  free(dz);
  return 0;
}

typedef struct {
  int Cin, H, W, Cout, KH, KW, stride, pad, groups, n, Ho, Wo, b0;
  const double *dy, *experts, *alpha, *dg;
  double *dx;   /* [nb][H][W][Cin] */
} dgrad_ctx;

static void dgrad_one(void *vctx, int b) {
  dgrad_ctx *f = (dgrad_ctx *)vctx;
  const int Cg = f->Cin / f->groups, Coutg = f->Cout / f->groups;
  const long wsize = (long)f->Cout * f->KH * f->KW * Cg;
  double *Wb = (double *)malloc(sizeof(double) * (size_t)wsize);
  oracle_assemble(f->n, wsize, f->experts, f->alpha + (size_t)b * f->n, Wb);
  double *dxb = f->dx + (size_t)(b - f->b0) * f->H * f->W * f->Cin;
  memset(dxb, 0, sizeof(double) * (size_t)f->H * f->W * f->Cin);
  const double *dyb = f->dy + (size_t)b * f->Ho * f->Wo * f->Cout;
  for (int oh = 0; oh < f->Ho; ++oh)
    for (int ow = 0; ow < f->Wo; ++ow)
      for (int co = 0; co < f->Cout; ++co) {
        const double d = dyb[((size_t)oh * f->Wo + ow) * f->Cout + co];
        const size_t cin0 = (size_t)(co / Coutg) * Cg;
        for (int kh = 0; kh < f->KH; ++kh)
          for (int kw = 0; kw < f->KW; ++kw) {
            const int y_in = f->stride * oh - f->pad + kh, x_in = f->stride * ow - f->pad + kw;
            if (y_in < 0 || y_in >= f->H || x_in < 0 || x_in >= f->W) continue;  /* padding */
            double *gx = dxb + ((size_t)y_in * f->W + x_in) * f->Cin + cin0;
            const double *wv = Wb + ((size_t)(co * f->KH + kh) * f->KW + kw) * Cg;
            for (int ci = 0; ci < Cg; ++ci) gx[ci] += d * wv[ci];
          }
      }
  if (f->dg) {
    const double *dgb = f->dg + (size_t)b * f->Cin;
    const double inv = 1.0 / (double)(f->H * f->W);
    for (long p = 0; p < (long)f->H * f->W; ++p)
      for (int c = 0; c < f->Cin; ++c) dxb[(size_t)p * f->Cin + c] += dgb[c] * inv;
  }
  free(Wb);
}

/* dx[nb][H][W][Cin] for samples b0 .. b0+nb-1: the convolution's input
 * gradient with the mixed kernel W_b, plus dg[b,c]/(H*W) on every pixel when
 * dg [B][Cin] is given (the pooled vector's gradient; NULL: none). */
int oracle_backward_data(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                         int pad, int groups, int n, const double *dy, const double *experts,
                         const double *alpha, const double *dg, int b0, int nb, double *dx,
                         int nthreads) {
  if (!bwd_shape_ok(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n)) return -1;
  if (!dy || !experts || !alpha || !dx || b0 < 0 || nb < 0 || b0 + nb > B) return -1;
  if (nb == 0) return 0;
  dgrad_ctx f = {Cin, H, W, Cout, KH, KW, stride, pad, groups, n,
                 oracle_out_size(H, KH, stride, pad), oracle_out_size(W, KW, stride, pad), b0,
                 dy, experts, alpha, dg, dx};
  return run_samples(dgrad_one, &f, b0, nb, nthreads);
}

/* ------------------------------------------------ restrictions for spot checks
 * The same definitions as oracle_backward_weight, restricted so that large
 * layers can be checked without holding every sample's gradient: dalpha of a
 * range of samples, dexperts at chosen weight elements, and dbias. */

typedef struct {
  int Cin, H, W, Cout, KH, KW, stride, pad, groups, n;
  const double *x, *dy, *experts, *bias;
  double *dalpha;   /* [nb][n] */
  int b0;
} dalpha_ctx;

static void dalpha_one(void *vctx, int b) {
  dalpha_ctx *f = (dalpha_ctx *)vctx;
  const long wsize = (long)f->Cout * f->KH * f->KW * (f->Cin / f->groups);
  double *dW = (double *)malloc(sizeof(double) * (size_t)wsize);
  double *db = (double *)malloc(sizeof(double) * (size_t)f->Cout);
  wgrad_ctx w = {f->Cin, f->H, f->W, f->Cout, f->KH, f->KW, f->stride, f->pad, f->groups,
                 oracle_out_size(f->H, f->KH, f->stride, f->pad),
                 oracle_out_size(f->W, f->KW, f->stride, f->pad), b, f->x, f->dy, dW, db};
  wgrad_one(&w, b);
  for (int i = 0; i < f->n; ++i) {
    double s = 0.0;
    for (long e = 0; e < wsize; ++e) s += dW[e] * f->experts[(size_t)i * wsize + e];
    if (f->bias)
      for (int co = 0; co < f->Cout; ++co) s += db[co] * f->bias[(size_t)i * f->Cout + co];
    f->dalpha[(size_t)(b - f->b0) * f->n + i] = s;
  }
  free(dW);
  free(db);
}

/* dalpha[nb][n] of samples b0 .. b0+nb-1. */
int oracle_dalpha(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride, int pad,
                  int groups, int n, const double *x, const double *dy, const double *experts,
                  const double *bias, int b0, int nb, double *dalpha, int nthreads) {
  if (!bwd_shape_ok(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n)) return -1;
  if (!x || !dy || !experts || !dalpha || b0 < 0 || nb < 0 || b0 + nb > B) return -1;
  if (nb == 0) return 0;
  dalpha_ctx f = {Cin, H, W, Cout, KH, KW, stride, pad, groups, n, x, dy, experts, bias, dalpha, b0};
  return run_samples(dalpha_one, &f, b0, nb, nthreads);
}

/* dexperts[i][idx[k]] for the flat weight indices idx[0 .. nidx-1] (layout
 * [C_out][KH][KW][C_in/groups]), written to out[n][nidx]: the per-sample
 * gradient of that one weight, summed over samples in order with alpha. */
int oracle_dexperts_at(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                       int pad, int groups, int n, const double *x, const double *dy,
                       const double *alpha, int nidx, const long *idx, double *out) {
  if (!bwd_shape_ok(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n)) return -1;
  if (!x || !dy || !alpha || !idx || !out || nidx < 0) return -1;
  const int Cg = Cin / groups, Coutg = Cout / groups;
  const int Ho = oracle_out_size(H, KH, stride, pad), Wo = oracle_out_size(W, KW, stride, pad);
  const long wsize = (long)Cout * KH * KW * Cg;
  for (int k = 0; k < nidx; ++k) {
    const long e = idx[k];
    if (e < 0 || e >= wsize) return -1;
    const int cil = (int)(e % Cg);
    const int kw = (int)((e / Cg) % KW), kh = (int)((e / Cg / KW) % KH);
    const int co = (int)(e / Cg / KW / KH);
    const int ci = (co / Coutg) * Cg + cil;
    for (int i = 0; i < n; ++i) out[(size_t)i * nidx + k] = 0.0;
    for (int b = 0; b < B; ++b) {
      double g = 0.0;
      for (int oh = 0; oh < Ho; ++oh)
        for (int ow = 0; ow < Wo; ++ow) {
          const int y_in = stride * oh - pad + kh, x_in = stride * ow - pad + kw;
          if (y_in < 0 || y_in >= H || x_in < 0 || x_in >= W) continue;
          g += dy[(((size_t)b * Ho + oh) * Wo + ow) * Cout + co] *
               x[(((size_t)b * H + y_in) * W + x_in) * Cin + ci];
        }
      for (int i = 0; i < n; ++i) out[(size_t)i * nidx + k] += alpha[(size_t)b * n + i] * g;
    }
  }
  return 0;
}

/* dbias[n][Cout] = sum_b alpha[b][i] * (sum over output pixels of dy[b][.][.][co]). */
int oracle_dbias(int B, int HoWo, int Cout, int n, const double *dy, const double *alpha,
                 double *dbias) {
  if (B < 0 || HoWo <= 0 || Cout <= 0 || n <= 0 || !dy || !alpha || !dbias) return -1;
  double *db = (double *)malloc(sizeof(double) * (size_t)Cout);
  if (!db) return -1;
  memset(dbias, 0, sizeof(double) * (size_t)n * Cout);
  for (int b = 0; b < B; ++b) {
    for (int co = 0; co < Cout; ++co) db[co] = 0.0;
    for (long p = 0; p < HoWo; ++p)
      for (int co = 0; co < Cout; ++co) db[co] += dy[((size_t)b * HoWo + p) * Cout + co];
    for (int i = 0; i < n; ++i)
      for (int co = 0; co < Cout; ++co) dbias[(size_t)i * Cout + co] += alpha[(size_t)b * n + i] * db[co];
  }
  free(db);
  return 0;
}

/* =========================================================== kernel cells */
/*
 * Kernel cells shared through a warehouse (KernelWarehouse: Rethinking the
 * Design of Dynamic Convolution, abstract: the page redefines the kernel, its
 * assembly and the attention function so that n can exceed 100, by sharing
 * parameters within a layer and across neighbouring layers; it gives no
 * formula). Reading taken: the layer's kernel, flattened in the layout
 * [C_out][KH][KW][C_in/groups], is split into m contiguous cells of s
 * elements; a warehouse holds n cells E[n][s] (one warehouse may serve several
 * layers); every kernel cell j of sample b is its own mixture
 *     W_b[j*s + e] = sum_i alpha[b][j][i] * E[i][e],
 * with the attentions from the same router (average pool, one linear layer
 * with m*n outputs) normalised per cell: softmax over the n values of each
 * cell (z / tau), or an elementwise sigmoid. With m = 1 this is the ordinary
 * mixture of n kernels.
 */

/* W_b of one sample from its cell attentions alpha_b[m][n]. */
void oracle_assemble_cells(int m, int n, long s, const double *warehouse,
                           const double *alpha_b, double *Wb) {
  for (int j = 0; j < m; ++j)
    for (long e = 0; e < s; ++e) {
      double acc = 0.0;
      for (int i = 0; i < n; ++i) acc += alpha_b[(size_t)j * n + i] * warehouse[(size_t)i * s + e];
      Wb[(size_t)j * s + e] = acc;
    }
}

/* alpha[B][m][n]: the router with m*n outputs, its activation taken per cell. */
int oracle_route_cells(int B, int C, int H, int W, const double *x, int m, int n,
                       const double *Wr, const double *br, int mode, double tau, double *alpha) {
  if (B < 0 || C <= 0 || H <= 0 || W <= 0 || m <= 0 || n <= 0 || !x || !Wr || !alpha) return -1;
  if (mode != ORACLE_SIGMOID && mode != ORACLE_SOFTMAX) return -1;
  if (mode == ORACLE_SOFTMAX && !(tau > 0.0)) return -1;
  double *g = (double *)malloc(sizeof(double) * (size_t)C);
  double *z = (double *)malloc(sizeof(double) * (size_t)m * n);
  if (!g || !z) { free(g); free(z); return -1; }
  for (int b = 0; b < B; ++b) {
    oracle_gap(C, H, W, x + (size_t)b * H * W * C, g);
    oracle_fc(C, m * n, Wr, br, g, z);
    for (int j = 0; j < m; ++j)
      oracle_act(n, z + (size_t)j * n, mode, tau, alpha + ((size_t)b * m + j) * n);
  }
  free(g);
  free(z);
  return 0;
}

/* y of samples b0 .. b0+nb-1 with the kernel assembled from cells, plus an
 * optional static bias[C_out] (not mixed): the convolution is oracle_forward
 * of one sample with W_b as its only expert and attention 1. */
int oracle_forward_cells(int B, int Cin, int H, int W, int Cout, int KH, int KW, int stride,
                         int pad, int groups, int m, int n, const double *x,
                         const double *warehouse, const double *alpha, const double *bias,
                         int b0, int nb, double *y) {
  if (B < 0 || Cin <= 0 || H <= 0 || W <= 0 || Cout <= 0 || KH <= 0 || KW <= 0) return -1;
  if (m <= 0 || n <= 0 || groups <= 0 || Cin % groups || Cout % groups) return -1;
  if (!x || !warehouse || !alpha || !y || b0 < 0 || nb < 0 || b0 + nb > B) return -1;
  const long wsize = (long)Cout * KH * KW * (Cin / groups);
  if (wsize % m != 0) return -1;
  const long s = wsize / m;
  const int Ho = oracle_out_size(H, KH, stride, pad), Wo = oracle_out_size(W, KW, stride, pad);
  if (Ho <= 0 || Wo <= 0) return -1;
  double *Wb = (double *)malloc(sizeof(double) * (size_t)wsize);
  if (!Wb) return -1;
  const double one = 1.0;
  int rc = 0;
  for (int b = b0; b < b0 + nb && rc == 0; ++b) {
    oracle_assemble_cells(m, n, s, warehouse, alpha + (size_t)b * m * n, Wb);
    rc = oracle_forward(1, Cin, H, W, Cout, KH, KW, stride, pad, groups, 1,
                        x + (size_t)b * H * W * Cin, Wb, &one, bias, 0, 1,
                        y + (size_t)(b - b0) * Ho * Wo * Cout, 1);
  }
  free(Wb);
  return rc;
}
