/* Plain fp64 reduction of the W4A4 GEMM reference (oracle; test infrastructure only).
 *
 * y[m][n] = sum over k = 0, 1, ..., K-1 (in that order) of x[m][k] * w[n][k]
 * t[m][n] = the same sum of |x[m][k] * w[n][k]|        (the per-element tolerance scale)
 *
 * This is the definition of the quantized linear layer y = X W^T that the pages share (PRQuant,
 * §4 "Kernel design for efficient inference": one GEMM over the quantized operands; MXCode,
 * abstract: MX-native W4A4 operands), evaluated on the dequantized operands.  Every summand is
 * added to one running fp64 total in ascending k: no blocking, no reassociation, no library
 * matmul.  Built with -ffp-contract=off so no multiply-add is fused (the products of dequantized
 * FP4/INT4 operands are exact in fp64 anyway).  Output rows are independent and are shared out
 * over OpenMP threads; each element's sum is computed by one thread in the order above.
 * Four output columns are summed side by side only to keep the floating-point unit busy; each of
 * the four running totals still takes its own terms in ascending k.
 */
#include <math.h>
#include <stdint.h>

void oracle_gemm_nt(int64_t M, int64_t N, int64_t K, const double* x, const double* w,
                    double* y, double* t) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    const double* xr = x + m * K;
    int64_t n = 0;
    for (; n + 4 <= N; n += 4) {
      const double* w0 = w + (n + 0) * K;
      const double* w1 = w + (n + 1) * K;
      const double* w2 = w + (n + 2) * K;
      const double* w3 = w + (n + 3) * K;
      double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const double xv = xr[k];
        const double p0 = xv * w0[k], p1 = xv * w1[k], p2 = xv * w2[k], p3 = xv * w3[k];
        s0 += p0; s1 += p1; s2 += p2; s3 += p3;
        a0 += fabs(p0); a1 += fabs(p1); a2 += fabs(p2); a3 += fabs(p3);
      }
      y[m * N + n + 0] = s0; y[m * N + n + 1] = s1; y[m * N + n + 2] = s2; y[m * N + n + 3] = s3;
      if (t) {
        t[m * N + n + 0] = a0; t[m * N + n + 1] = a1; t[m * N + n + 2] = a2; t[m * N + n + 3] = a3;
      }
    }
    for (; n < N; ++n) {
      const double* wr = w + n * K;
      double s = 0.0, a = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const double p = xr[k] * wr[k];
        s += p;
        a += fabs(p);
      }
      y[m * N + n] = s;
      if (t) t[m * N + n] = a;
    }
  }
}
