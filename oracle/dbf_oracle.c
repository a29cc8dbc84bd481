/*
 * fp64 CPU oracle for the Double Binary Factorization (DBF) layer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, __graft_entry__.smoke()
 * and bench.py's cpu_baseline / reference leg may load this library.  It shares
 * no source, header, table or helper with the CUDA path in
 * binary_factorized_weight_b200/ and neither side includes or calls the other.
 *
 * Source: "Addition is almost all you need: Compressing large language models
 * with double binary factorization" (gist.science technical summary, section
 * 2.1 "mathematical formulation"; sciencestack.ai abstract and Figure 1).
 *
 *   factorisation  W ~= (a (.) A (.) m^T)(B (.) b^T),  A in {+-1}^(n x k),
 *                  B in {+-1}^(k x m_in), a, m, b fp16 vectors   (section 2.1)
 *   evaluation     X W^T ~= ((((X (.) b^T) B^T) (.) m^T) A^T) (.) a^T
 *                  every product with a sign matrix is additions and sign
 *                  flips                                      (section 2.1,
 *                                                  "computation process")
 *
 * Everything is computed in fp64 from inputs that the caller has widened
 * exactly from fp16 / +-1.  The method has no approximation at inference time,
 * so the oracle is the plain definition written out with loops; no blocking,
 * fusion or reordering beyond the evaluation order above.
 *
 * Packed sign layout decoded by oracle_unpack_signs (the pages only say the
 * matrices are binary/sign; the bit layout is this library's own choice):
 *   - a rows x cols sign matrix is stored row after row; each row takes
 *     ceil(cols/256)*8 little-endian 32-bit words (a multiple of 32 bytes),
 *     one block of 8 words per 256 columns;
 *   - inside a block, column e (0..255) belongs to group g = e/16 and pair
 *     p = (e%16)/2 of that group; it is held in word p of the block, at bit
 *     g + 16*(e%2).  So word p carries pair p of all 16 groups, even columns
 *     in bits 0..15 and odd columns in bits 16..31;
 *   - a set bit means -1, a clear bit +1; bits past the last column are 0.
 *
 * Parity status of each function (see the test-suite pins in
 * tests/test_oracle_pins.py):
 *   oracle_forward_staged, oracle_forward_transposed, oracle_dense_weight,
 *   oracle_forward_dense, oracle_unpack_signs, oracle_pack_signs,
 *   oracle_bits_per_weight, oracle_scale_bits_per_weight, oracle_bqq_dense_weight:
 *   pinned.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads for the parallel loops below (timing only; results do not depend on it). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Words per packed row: the row is padded to a multiple of 256 columns. */
int64_t oracle_words_per_row(int64_t cols) { return ((cols + 255) / 256) * 8; }

/* Word (within the row) and bit holding column c. */
static int64_t word_of_column(int64_t c) { return (c / 256) * 8 + (c % 16) / 2; }
static int bit_of_column(int64_t c) { return (int)((c % 256) / 16) + 16 * (int)(c % 2); }

/*
 * Decode a packed sign matrix into int8 +-1 values (row-major rows x cols).
 * Returns the number of set padding bits found (0 for a valid buffer).
 */
int64_t oracle_unpack_signs(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* out) {
  const int64_t wpr = oracle_words_per_row(cols);
  int64_t bad_padding = 0;
  for (int64_t r = 0; r < rows; ++r) {
    const uint32_t* row = packed + r * wpr;
    for (int64_t c = 0; c < cols; ++c) {
      uint32_t word = row[word_of_column(c)];
      out[r * cols + c] = ((word >> bit_of_column(c)) & 1u) ? (int8_t)-1 : (int8_t)1;
    }
    for (int64_t c = cols; c < wpr * 32; ++c) {
      uint32_t word = row[word_of_column(c)];
      bad_padding += (word >> bit_of_column(c)) & 1u;
    }
  }
  return bad_padding;
}

/*
 * Encode int8 signs into the packed layout.  An entry < 0 becomes a set bit;
 * 0 and positive entries become clear bits.
 */
void oracle_pack_signs(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* packed) {
  const int64_t wpr = oracle_words_per_row(cols);
  memset(packed, 0, (size_t)(rows * wpr) * sizeof(uint32_t));
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      if (signs[r * cols + c] < 0) {
        packed[r * wpr + word_of_column(c)] |= 1u << bit_of_column(c);
      }
    }
  }
}

/*
 * Staged forward, in the order of the "computation process" equation:
 *   u = x (.) b                (X (.) b^T)
 *   t = B u                    (. B^T, additions and sign flips)
 *   v = mid (.) t              ((.) m^T)
 *   z = A v                    (. A^T, additions and sign flips)
 *   y = a (.) z                ((.) a^T)
 * x is batch x m_in, y is batch x n, A is n x k, B is k x m_in (row-major int8).
 * If v_out is non-NULL it receives v (batch x k).
 */
void oracle_forward_staged(const double* x, const int8_t* A, const int8_t* B, const double* a,
                           const double* mid, const double* b, int64_t n, int64_t k, int64_t m_in,
                           int64_t batch, double* y, double* v_out) {
  double* ubuf = (double*)malloc((size_t)m_in * sizeof(double));
  double* vbuf = (double*)malloc((size_t)k * sizeof(double));
  if (!ubuf || !vbuf) {
    free(ubuf);
    free(vbuf);
    for (int64_t e = 0; e < batch * n; ++e) y[e] = NAN;
    return;
  }
  for (int64_t tok = 0; tok < batch; ++tok) {
    const double* xt = x + tok * m_in;
    for (int64_t j = 0; j < m_in; ++j) ubuf[j] = xt[j] * b[j];
#pragma omp parallel for schedule(static)
    for (int64_t l = 0; l < k; ++l) {
      const int8_t* Bl = B + l * m_in;
      double acc = 0.0;
      for (int64_t j = 0; j < m_in; ++j) acc += (double)Bl[j] * ubuf[j];
      vbuf[l] = mid[l] * acc;
    }
    if (v_out) memcpy(v_out + tok * k, vbuf, (size_t)k * sizeof(double));
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
      const int8_t* Ai = A + i * k;
      double acc = 0.0;
      for (int64_t l = 0; l < k; ++l) acc += (double)Ai[l] * vbuf[l];
      y[tok * n + i] = a[i] * acc;
    }
  }
  free(ubuf);
  free(vbuf);
}

/* The transpose product dx = dy W for the factorised W (section 2.1: W is
 * n x m_in with y = x W^T, so dy W is the product with W^T's transpose, the
 * input gradient of the layer).  With W = (a (.) A (.) mid^T)(B (.) b^T):
 *     dx[t][j] = b_j * sum_l B[l][j] * mid_l * sum_i A[i][l] * a_i * dy[t][i],
 * evaluated right to left like the forward, without forming W.
 * dy: batch x n; dx: batch x m_in.  fp64 throughout. */
void oracle_forward_transposed(const double* dy, const int8_t* A, const int8_t* B, const double* a,
                               const double* mid, const double* b, int64_t n, int64_t k, int64_t m_in,
                               int64_t batch, double* dx) {
  double* gbuf = (double*)malloc((size_t)n * sizeof(double));
  double* vbuf = (double*)malloc((size_t)k * sizeof(double));
  if (!gbuf || !vbuf) {
    free(gbuf);
    free(vbuf);
    for (int64_t e = 0; e < batch * m_in; ++e) dx[e] = NAN;
    return;
  }
  for (int64_t tok = 0; tok < batch; ++tok) {
    const double* dyt = dy + tok * n;
    for (int64_t i = 0; i < n; ++i) gbuf[i] = a[i] * dyt[i];
#pragma omp parallel for schedule(static)
    for (int64_t l = 0; l < k; ++l) {
      double acc = 0.0;
      for (int64_t i = 0; i < n; ++i) acc += (double)A[i * k + l] * gbuf[i];
      vbuf[l] = mid[l] * acc;
    }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < m_in; ++j) {
      double acc = 0.0;
      for (int64_t l = 0; l < k; ++l) acc += (double)B[l * m_in + j] * vbuf[l];
      dx[tok * m_in + j] = b[j] * acc;
    }
  }
  free(gbuf);
  free(vbuf);
}

/*
 * Dense reconstruction W = (a (.) A (.) m^T)(B (.) b^T), n x m_in:
 *   W[i][j] = sum_l (a_i A[i][l] m_l) (B[l][j] b_j)
 */
void oracle_dense_weight(const int8_t* A, const int8_t* B, const double* a, const double* mid,
                         const double* b, int64_t n, int64_t k, int64_t m_in, double* W) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    double* Wi = W + i * m_in;
    for (int64_t j = 0; j < m_in; ++j) Wi[j] = 0.0;
    for (int64_t l = 0; l < k; ++l) {
      const double left = a[i] * (double)A[i * k + l] * mid[l];
      const int8_t* Bl = B + l * m_in;
      for (int64_t j = 0; j < m_in; ++j) Wi[j] += left * ((double)Bl[j] * b[j]);
    }
  }
}

/*
 * Binary Quadratic Quantization (sciencestack.ai page of "Binary Quadratic
 * Quantization: Beyond First-Order Quantization for Real-Valued Matrix
 * Compression", TL;DR formula):
 *     W = sum_{i<p} (r_i Y_i Z_i + s_i Y_i 1_Z + t_i 1_Y Z_i) + u 1,
 * with binary Y_i (n x k) and Z_i (k x m), real scalars r_i, s_i, t_i, u, and
 * 1_Z, 1_Y, 1 all-ones matrices of the shapes of Z_i, Y_i and W.  The binary
 * alphabet is read as {0, 1} (the page builds on polynomial unconstrained
 * binary optimisation).  Y holds the p matrices Y_i one after the other
 * (p x n x k, row-major), Z likewise (p x k x m); entries 0 or 1.
 *     (Y_i 1_Z)[a][c] = sum_l Y_i[a][l]       (1_Z is k x m)
 *     (1_Y Z_i)[a][c] = sum_l Z_i[l][c]       (1_Y is n x k)
 */
void oracle_bqq_dense_weight(const int8_t* Y, const int8_t* Z, const double* r, const double* s, const double* t,
                             double u, int64_t n, int64_t k, int64_t m, int64_t p, double* W) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    for (int64_t c = 0; c < m; ++c) {
      double w = u;
      for (int64_t i = 0; i < p; ++i) {
        const int8_t* Yi = Y + i * n * k;
        const int8_t* Zi = Z + i * k * m;
        double yz = 0.0, y_row = 0.0, z_col = 0.0;
        for (int64_t l = 0; l < k; ++l) {
          yz += (double)Yi[a * k + l] * (double)Zi[l * m + c];
          y_row += (double)Yi[a * k + l];
          z_col += (double)Zi[l * m + c];
        }
        w += r[i] * yz;
        w += s[i] * y_row;
        w += t[i] * z_col;
      }
      W[a * m + c] = w;
    }
  }
}

/* y = x W^T for a dense W (n x m_in); x is batch x m_in. */
void oracle_forward_dense(const double* x, const double* W, int64_t n, int64_t m_in, int64_t batch,
                          double* y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t tok = 0; tok < batch; ++tok) {
    for (int64_t i = 0; i < n; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < m_in; ++j) acc += x[tok * m_in + j] * W[i * m_in + j];
      y[tok * n + i] = acc;
    }
  }
}

/*
 * Storage cost.  Section 2.1 names the middle dimension k as the knob that
 * sets the compression rate (section 2.3 builds the per-layer allocation on
 * it).  Sign bits per dense weight: k(n + m_in)/(n m_in).
 * The three fp16 scale vectors add 16(n + k + m_in)/(n m_in).
 */
double oracle_bits_per_weight(int64_t n, int64_t k, int64_t m_in) {
  return (double)k * (double)(n + m_in) / ((double)n * (double)m_in);
}

double oracle_scale_bits_per_weight(int64_t n, int64_t k, int64_t m_in) {
  return 16.0 * (double)(n + k + m_in) / ((double)n * (double)m_in);
}
