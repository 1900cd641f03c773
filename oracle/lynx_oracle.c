/*
 * lynx_oracle.c -- plain, slow, obviously-correct CPU oracle for the RT-Lynx
 * online 2:4 activation-sparse linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (sources are the pages about "RT-Lynx: Putting GEMM
 * Sparsity in the Right Place for Diffusion Models"):
 *
 *   Y = S(X) W^T + bias + (X A^T) B^T
 *
 *   - qingkeai.online article, section 02 ("why activations"): the linear
 *     layer becomes Y = S(X) W^T, S(X) a 2:4 pattern generated at run time.
 *   - ai-feeds.com summary, "input and sparsification strategy": in every 4
 *     consecutive values 2 are kept; neuraltrendhub summary: "N:M" applied
 *     token-wise.  Selection is Top-K by magnitude (qingkeai section 03).
 *     Ties go to the lower index (the pages are silent; plainest reading).
 *   - ai-feeds.com "core module 1" and qingkeai section 03.1 (norm
 *     compensation): the pruned L1 mass is handed back to the kept values in
 *     proportion.  v + P*|v|/L_kept*sign(v) = v * L_all / L_kept, so it is a
 *     per-token-row factor s = sum|x| / sum|kept| (s := 1 if nothing kept has
 *     non-zero magnitude), computed in fp32 and applied to the kept values,
 *     which are rounded once to bf16.
 *   - qingkeai section 03.2 (LoRA compensation): a low-rank branch on the
 *     frozen backbone restores the fine residual; neuraltrendhub: rank 64.
 *     It is taken on the dense X, with no extra alpha/r factor (folded into B).
 *   - qingkeai section 03.3 (selective layer skipping): skipped layers stay
 *     dense, S(X) := X.
 *
 *   - An activation on the layer's output (not part of the pages' method; the
 *     DiT MLP applies it between its up- and down-projections, and the
 *     library can apply it in the GEMM epilogue): GELU, tanh form
 *     (Hendrycks & Gimpel, "Gaussian Error Linear Units"),
 *     gelu(v) = v/2 (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), in fp64.
 *
 * Precision: selection compares magnitudes exactly; the two row sums are fp32
 * sums in increasing k order; s is one IEEE fp32 division; each kept value is
 * one fp32 multiply rounded to nearest even, then rounded to nearest even to
 * bf16.  All dot products (T, Y) are accumulated in fp64 from the bf16 inputs.
 *
 * Canonical metadata format (the comparison format, not the GPU's operand
 * layout): row m owns K/8 bytes; group g (k = 4g..4g+3) is the nibble
 * lo | hi << 2 (lo < hi, the two kept positions inside the group) in byte
 * m*K/8 + g/2, low nibble for even g.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (see build.py).
 * Floating point must not be contracted or reassociated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef uint16_t bf16_bits;

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static float bf16_to_f32(bf16_bits h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* IEEE round-to-nearest, ties-to-even, binary32 -> bf16 (finite inputs).
 * Keep the upper 16 bits; the discarded lower 16 bits are compared with half
 * a unit in the last kept place (0x8000).  Above half: round up.  Exactly
 * half: round up only if the kept part is odd.  An increment that carries
 * into the exponent field is the correct next binade by the IEEE encoding. */
static bf16_bits f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint32_t kept = u >> 16;
  uint32_t dropped = u & 0xFFFFu;
  if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
  return (bf16_bits)kept;
}

/* Top-2 of a group of 4 by magnitude, ties to the lower index.
 * First pick: the largest magnitude, scanning up and replacing only on a
 * strictly larger value, so the lowest index wins a tie.  Second pick: the
 * same scan over the three remaining positions. */
static void select_top2(const bf16_bits g[4], int *lo, int *hi) {
  float a[4];
  for (int i = 0; i < 4; ++i) a[i] = fabsf(bf16_to_f32(g[i]));
  int i0 = 0;
  for (int i = 1; i < 4; ++i)
    if (a[i] > a[i0]) i0 = i;
  int i1 = -1;
  for (int i = 0; i < 4; ++i) {
    if (i == i0) continue;
    if (i1 < 0 || a[i] > a[i1]) i1 = i;
  }
  *lo = i0 < i1 ? i0 : i1;
  *hi = i0 < i1 ? i1 : i0;
}

/* ---------------------------------------------------------------------- */
/* Exported helpers (used by the pin tests).                               */

void oracle_bf16_rne(const float *in, bf16_bits *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

/* groups: [n,4] bf16 bits -> lo[n], hi[n] */
void oracle_select_groups(const bf16_bits *groups, int64_t n, int32_t *lo, int32_t *hi) {
  for (int64_t i = 0; i < n; ++i) {
    int l, h;
    select_top2(groups + 4 * i, &l, &h);
    lo[i] = l;
    hi[i] = h;
  }
}

/* One token row of S(X).
 *   x        [K]     bf16 input row
 *   vals     [K/2]   kept values after compensation, ascending index order
 *   meta     [K/8]   canonical nibbles
 *   dense    [K]     S(X) row widened to double (NULL to skip)
 *   scale    s (fp32); l_all32/l_kept32 the fp32 sums; l_all64/l_kept64 the
 *            same sums in fp64 (for invariant checks) */
static void sparsify_row(const bf16_bits *x, int64_t K, bf16_bits *vals, uint8_t *meta,
                         double *dense, float *scale, float *l_all32, float *l_kept32,
                         double *l_all64, double *l_kept64) {
  const int64_t G = K / 4;
  float la = 0.0f, lk = 0.0f;
  double la64 = 0.0, lk64 = 0.0;
  /* pass 1: decisions and the two sums, in increasing k order */
  for (int64_t g = 0; g < G; ++g) {
    int lo, hi;
    select_top2(x + 4 * g, &lo, &hi);
    for (int i = 0; i < 4; ++i) {
      float a = fabsf(bf16_to_f32(x[4 * g + i]));
      la += a;
      la64 += (double)a;
      if (i == lo || i == hi) {
        lk += a;
        lk64 += (double)a;
      }
    }
    uint8_t nib = (uint8_t)(lo | (hi << 2));
    if ((g & 1) == 0)
      meta[g / 2] = nib;
    else
      meta[g / 2] = (uint8_t)(meta[g / 2] | (nib << 4));
  }
  float s = (lk == 0.0f) ? 1.0f : la / lk;
  /* pass 2: compensated kept values */
  if (dense) memset(dense, 0, sizeof(double) * (size_t)K);
  for (int64_t g = 0; g < G; ++g) {
    uint8_t nib = (g & 1) ? (uint8_t)(meta[g / 2] >> 4) : (uint8_t)(meta[g / 2] & 0xF);
    int lo = nib & 3, hi = (nib >> 2) & 3;
    float p_lo = bf16_to_f32(x[4 * g + lo]) * s;
    float p_hi = bf16_to_f32(x[4 * g + hi]) * s;
    bf16_bits v_lo = f32_to_bf16_rne(p_lo);
    bf16_bits v_hi = f32_to_bf16_rne(p_hi);
    vals[2 * g] = v_lo;
    vals[2 * g + 1] = v_hi;
    if (dense) {
      dense[4 * g + lo] = (double)bf16_to_f32(v_lo);
      dense[4 * g + hi] = (double)bf16_to_f32(v_hi);
    }
  }
  *scale = s;
  if (l_all32) *l_all32 = la;
  if (l_kept32) *l_kept32 = lk;
  if (l_all64) *l_all64 = la64;
  if (l_kept64) *l_kept64 = lk64;
}

/* S(X) for a whole matrix.  X [M,K]; vals [M,K/2]; meta [M,K/8]; scale [M];
 * sums [M,4] (l_all32, l_kept32, l_all64, l_kept64) as doubles, may be NULL. */
void oracle_sparsify(const bf16_bits *X, int64_t M, int64_t K, bf16_bits *vals, uint8_t *meta,
                     float *scale, double *sums) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t m = 0; m < M; ++m) {
    float la32, lk32;
    double la64, lk64;
    sparsify_row(X + m * K, K, vals + m * (K / 2), meta + m * (K / 8), NULL, scale + m, &la32,
                 &lk32, &la64, &lk64);
    if (sums) {
      sums[4 * m + 0] = la32;
      sums[4 * m + 1] = lk32;
      sums[4 * m + 2] = la64;
      sums[4 * m + 3] = lk64;
    }
  }
}

/* The full layer, in fp64 from the bf16 inputs.
 *   X [M,K], W [N,K], bias [N] or NULL, A [r,K] and B [N,r] or both NULL.
 *   skip != 0: S(X) := X (a layer left dense by selective layer skipping).
 *   Y [M,N] (double, unrounded); T [M,r] (double) or NULL; SX [M,K] (double)
 *   or NULL receives the dense S(X) actually multiplied. */
void oracle_linear(const bf16_bits *X, const bf16_bits *W, const bf16_bits *bias,
                   const bf16_bits *A, const bf16_bits *B, int64_t M, int64_t N, int64_t K,
                   int64_t r, int skip, double *Y, double *T, double *SX) {
  const int lora = (A != NULL && B != NULL && r > 0);
#pragma omp parallel
  {
    double *srow = (double *)malloc(sizeof(double) * (size_t)K);
    double *trow = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
    bf16_bits *vrow = (bf16_bits *)malloc(sizeof(bf16_bits) * (size_t)(K / 2 + 1));
    uint8_t *mrow = (uint8_t *)malloc((size_t)(K / 8 + 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
      const bf16_bits *x = X + m * K;
      if (skip) {
        for (int64_t k = 0; k < K; ++k) srow[k] = (double)bf16_to_f32(x[k]);
      } else {
        float s;
        sparsify_row(x, K, vrow, mrow, srow, &s, NULL, NULL, NULL, NULL);
      }
      if (SX)
        for (int64_t k = 0; k < K; ++k) SX[m * K + k] = srow[k];
      if (lora) {
        for (int64_t j = 0; j < r; ++j) {
          double acc = 0.0;
          for (int64_t k = 0; k < K; ++k)
            acc += (double)bf16_to_f32(x[k]) * (double)bf16_to_f32(A[j * K + k]);
          trow[j] = acc;
          if (T) T[m * r + j] = acc;
        }
      }
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        const bf16_bits *w = W + n * K;
        for (int64_t k = 0; k < K; ++k) acc += srow[k] * (double)bf16_to_f32(w[k]);
        if (bias) acc += (double)bf16_to_f32(bias[n]);
        if (lora)
          for (int64_t j = 0; j < r; ++j) acc += trow[j] * (double)bf16_to_f32(B[n * r + j]);
        Y[m * N + n] = acc;
      }
    }
    free(srow);
    free(trow);
    free(vrow);
    free(mrow);
  }
}

/* GELU, tanh form, in fp64, for n values.  Written with the identity
 * (1 + tanh u)/2 = 1/(1 + exp(-2u)), the same function without the
 * cancellation in 1 + tanh u when u is very negative. */
void oracle_gelu_tanh(const double *v, int64_t n, double *out) {
  const double c = sqrt(2.0 / 3.14159265358979323846);
  for (int64_t i = 0; i < n; ++i) {
    const double x = v[i];
    const double u = c * (x + 0.044715 * x * x * x);
    out[i] = x / (1.0 + exp(-2.0 * u));
  }
}

/* Threads used by the parallel loops above from now on (timing only; the
 * results do not depend on it: every output element is computed by one thread
 * in a fixed order). */
void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
