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
 *   routing   alpha_b = act(FC(GAP(x_b)))  -- "input-dependent attentions"
 *             (KernelWarehouse: Rethinking the Design of Dynamic Convolution,
 *             abstract), one attention vector per example (CondConv:
 *             Conditionally Parameterized Convolutions for Efficient Inference,
 *             abstract); the temperature divides the logits before the softmax
 *             ("temperature-degraded kernel attention", FMDConv: Fast
 *             multi-attention dynamic convolution via speed-accuracy trade-off,
 *             abstract). The GAP -> single linear layer -> sigmoid/softmax form
 *             is the reading taken where the pages are silent.
 *   assembly  W_b = sum_i alpha_{b,i} W_i, b_b = sum_i alpha_{b,i} bias_i
 *             ("a linear mixture of n static kernels weighted with their
 *             input-dependent attentions", KernelWarehouse abstract).
 *   conv      y_b = conv2d(x_b, W_b) + b_b, cross-correlation with zero padding
 *             ("specialized convolutional kernels for each example", CondConv
 *             abstract); orientation and padding are readings, pinned by tests.
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
