/*
 * MapFlow hot-path oracle: a plain, slow, double-precision CPU statement of what
 * block-sparse attention-map compression and fused map retrieval compute.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load it; the library never does.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * Sources (MapFlow pages: "MapFlow开源:大模型换班,Prefill为何能快20%?",
 * aitest123.com, section "存不下、读得慢?三个工程优化手段", and its English
 * rendering on roboind.com, section "When it comes to real savings in reuse"):
 *   1. block-sparse compression: the map is cut into regular 2-D blocks and
 *      the important ones are chosen by cumulative attention probability;
 *      block statistics are computed first, then the blocks to keep are chosen
 *      (subsection 1 "只存重要的:块稀疏压缩").
 *   2. fused retrieval: read the sparse blocks, form the linear combination of
 *      sender heads into receiver heads, multiply by the receiver's own V and
 *      accumulate (subsection 3 "算得省的:融合内核执行"); the receiver keeps its
 *      own Value ("不传 KV Cache,改传注意力关系"); heads are mapped by learned
 *      linear-combination weights (same section, "头映射").
 *
 * Readings taken where the pages are silent:
 *   - selection is per query block on the head-summed mass, one index set for
 *     all heads; the diagonal block is always kept and counts toward tau;
 *   - the other key blocks are walked in (mass descending, index ascending)
 *     order; the walk keeps the fewest blocks whose running sum S reaches
 *     tau * total, where total is the sum of all the row's masses taken in the
 *     same walk order (so at tau = 1 the walk stops where S stops growing);
 *   - entries with j > i, i >= L or j >= L are 0 in the stored blocks and do not
 *     count toward any mass;
 *   - kept blocks are stored raw (no renormalisation), col_idx ascending;
 *   - receiver head r reads KV head g(r) = floor(r * h_kv / h_r).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* dtype codes: 0 = float32, 1 = bfloat16 (stored as its upper 16 bits), 2 = float64. */
static double value_at(const void* p, int dtype, int64_t idx) {
  if (dtype == 0) return (double)((const float*)p)[idx];
  if (dtype == 2) return ((const double*)p)[idx];
  uint32_t bits = (uint32_t)((const uint16_t*)p)[idx] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/*
 * Block statistics of one query-block row (compression, step 1).
 * slab: the rows [qb*B, qb*B + B) of every sender head; element (s, ii, j) at
 * s*head_stride + ii*row_stride + j.  mass[kb] for kb = 0..qb.
 */
void mfo_row_masses(const void* slab, int dtype, int h_s, int B, int64_t head_stride,
                    int64_t row_stride, int qb, int L, double* mass) {
  for (int kb = 0; kb <= qb; ++kb) {
    double m = 0.0;
    for (int s = 0; s < h_s; ++s)
      for (int ii = 0; ii < B; ++ii) {
        const int i = qb * B + ii;
        if (i >= L) break;
        for (int jj = 0; jj < B; ++jj) {
          const int j = kb * B + jj;
          if (j >= L || j > i) continue;
          m += value_at(slab, dtype, s * head_stride + ii * row_stride + j);
        }
      }
    mass[kb] = m;
  }
}

/* walk order of a row: the diagonal first, then kb < qb by (mass desc, kb asc). */
static void walk_order(const double* mass, int qb, int32_t* order) {
  int n = 0;
  order[n++] = qb;
  for (int kb = 0; kb < qb; ++kb) {
    /* insertion into order[1..n) */
    int p = n;
    while (p > 1) {
      const int o = order[p - 1];
      const int before = mass[kb] > mass[o] || (mass[kb] == mass[o] && kb < o);
      if (!before) break;
      order[p] = o;
      --p;
    }
    order[p] = kb;
    ++n;
  }
}

/*
 * Block selection of one row (compression, step 2).  Writes the kept key-block
 * indices ascending into kept[] and returns their count.  Optionally reports the
 * row total, the running sum after the last kept block and before it, and the
 * masses of the last kept and first dropped candidate (for boundary accounting;
 * -1 where there is none).
 */
int mfo_select(const double* mass, int qb, double tau, int32_t* kept, double* info /*[5] or NULL*/) {
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(qb + 1));
  walk_order(mass, qb, order);
  double total = 0.0;
  for (int k = 0; k <= qb; ++k) total += mass[order[k]];
  const double target = tau * total;
  double S = 0.0, S_prev = 0.0;
  int n_keep = qb + 1;
  for (int k = 0; k <= qb; ++k) {
    S_prev = S;
    S += mass[order[k]];
    if (S >= target) {
      n_keep = k + 1;
      break;
    }
  }
  if (info) {
    info[0] = total;
    info[1] = S;
    info[2] = n_keep >= 2 ? S_prev : -1.0;
    info[3] = n_keep >= 2 ? mass[order[n_keep - 1]] : -1.0;
    info[4] = n_keep <= qb ? mass[order[n_keep]] : -1.0;
  }
  /* ascending copy */
  int n = 0;
  for (int kb = 0; kb <= qb; ++kb)
    for (int k = 0; k < n_keep; ++k)
      if (order[k] == kb) {
        kept[n++] = kb;
        break;
      }
  free(order);
  return n_keep;
}

/*
 * Kept-block write (compression, step 3): out[s][ii][jj] = A_s[qb*B+ii][kb*B+jj]
 * where that entry is causal and inside the sequence, else 0.  out has the input
 * dtype; the copy is exact.
 */
void mfo_gather_block(const void* slab, int dtype, int h_s, int B, int64_t head_stride,
                      int64_t row_stride, int qb, int kb, int L, void* out) {
  for (int s = 0; s < h_s; ++s)
    for (int ii = 0; ii < B; ++ii)
      for (int jj = 0; jj < B; ++jj) {
        const int i = qb * B + ii, j = kb * B + jj;
        const int64_t o = ((int64_t)s * B + ii) * B + jj;
        const int keep = i < L && j < L && j <= i;
        const int64_t src = s * head_stride + ii * row_stride + j;
        if (dtype == 0)
          ((float*)out)[o] = keep ? ((const float*)slab)[src] : 0.0f;
        else if (dtype == 2)
          ((double*)out)[o] = keep ? ((const double*)slab)[src] : 0.0;
        else
          ((uint16_t*)out)[o] = keep ? ((const uint16_t*)slab)[src] : (uint16_t)0;
      }
}

/* where the receiver's V row of one key token lives (contiguous or paged). */
typedef struct {
  const void* V;               /* contiguous: [T, h_kv, d]; paged: [pages, page_size, h_kv, d] */
  int dtype;                   /* 0 f32, 1 bf16 */
  int paged, page_size;
  const int32_t* block_table;  /* paged: this sequence's page list */
  int64_t k_start;             /* contiguous: first token of this sequence in V */
  int h_kv, d;
} mfo_vref;

static int64_t v_offset(const mfo_vref* v, int64_t tok, int g) {
  if (v->paged) {
    const int64_t page = v->block_table[tok / v->page_size];
    return ((page * v->page_size + tok % v->page_size) * v->h_kv + g) * (int64_t)v->d;
  }
  return ((v->k_start + tok) * v->h_kv + g) * (int64_t)v->d;
}

/*
 * Fused retrieval of one query block (retrieval, all steps), for block-local rows
 * [i0, i1) of query block qb (the caller passes rows inside the sequence only).
 * vals: the row's kept blocks [n][h_s][B][B] with key-block indices kb[n];
 * W: [h_r][h_s] float32 of this receiver layer.  For each row i and receiver head r:
 *   P_r[i, j] = sum_s W[r, s] * A_s[i, j]     over the keys j <= i of the kept blocks
 *   O[i, r, :] = sum_j P_r[i, j] * V[j, g(r), :]
 * O: [(i1 - i0)][h_r][d] double.
 */
void mfo_retrieve_block(const void* vals, int dtype, const int32_t* kb, int n, int qb, int B,
                        int h_s, const float* W, int h_r, const mfo_vref* vref, int i0, int i1,
                        double* O) {
  const int d = vref->d;
  double* P = (double*)malloc(sizeof(double) * (size_t)n * B);
  for (int ii = i0; ii < i1; ++ii)
    for (int r = 0; r < h_r; ++r) {
      const int g = (int)(((int64_t)r * vref->h_kv) / h_r);
      for (int t = 0; t < n; ++t)
        for (int jj = 0; jj < B; ++jj) {
          double p = 0.0;
          for (int s = 0; s < h_s; ++s)
            p += (double)W[r * h_s + s] *
                 value_at(vals, dtype, (((int64_t)t * h_s + s) * B + ii) * B + jj);
          P[t * B + jj] = p;
        }
      double* o = O + ((int64_t)(ii - i0) * h_r + r) * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      const int64_t i = (int64_t)qb * B + ii;
      for (int t = 0; t < n; ++t)
        for (int jj = 0; jj < B; ++jj) {
          const double p = P[t * B + jj];
          if ((int64_t)kb[t] * B + jj > i) continue; /* not a causal key of row i */
          const int64_t base = v_offset(vref, (int64_t)kb[t] * B + jj, g);
          for (int c = 0; c < d; ++c) o[c] += p * value_at(vref->V, vref->dtype, base + c);
        }
    }
  free(P);
}

/*
 * Head-map calibration (offline step of the head mapping).  The pages say the linear-
 * combination weights that map sender heads onto receiver heads are learned once, offline,
 * with both models frozen (page "MapFlow开源:大模型换班,Prefill为何能快20%?", section
 * "不传 KV Cache,改传“注意力关系”", head and layer mapping), but give no objective.  Reading taken: ordinary least squares
 * of each receiver head's map on the sender heads' maps over the causal positions of the
 * calibration sequences, with an optional ridge term:
 *   w_r = argmin_w  sum_{i < L, j <= i} (Y_r[i, j] - sum_s w[s] X_s[i, j])^2 + ridge * |w|^2.
 *
 * mfo_calib_gram accumulates, for one sequence, the Gram matrix of the stacked features
 * f = (X_0 .. X_{h_s-1}, Y_0 .. Y_{h_r-1}) at every causal position (i < L, j <= i) into
 * gram[F][F] (F = h_s + h_r, double).  X: [h_s][Lp][Lp], Y: [h_r][Lp][Lp] raw (dtype 0 f32,
 * 1 bf16); entries with j > i or in the padding are never read.
 */
void mfo_calib_gram(const void* X, const void* Y, int dtype, int h_s, int h_r, int L,
                    int64_t Lp, double* gram) {
  const int F = h_s + h_r;
  double* f = (double*)malloc(sizeof(double) * (size_t)F);
  for (int64_t i = 0; i < L; ++i)
    for (int64_t j = 0; j <= i; ++j) {
      for (int s = 0; s < h_s; ++s) f[s] = value_at(X, dtype, ((int64_t)s * Lp + i) * Lp + j);
      for (int r = 0; r < h_r; ++r) f[h_s + r] = value_at(Y, dtype, ((int64_t)r * Lp + i) * Lp + j);
      for (int a = 0; a < F; ++a)
        for (int b = 0; b < F; ++b) gram[a * F + b] += f[a] * f[b];
    }
  free(f);
}

/*
 * The least-squares solve from an accumulated Gram: G = gram[0:h_s][0:h_s] + ridge * I is
 * factored as L L^T (Cholesky, the textbook column algorithm); for every receiver head r the
 * right-hand side is c_r = gram[0:h_s][h_s + r], and w_r solves G w_r = c_r.  residual[r] is
 * sum (Y_r - w_r . X)^2 = gram[h_s+r][h_s+r] - 2 w_r . c_r + w_r^T G0 w_r with G0 the Gram
 * without the ridge term.  W: [h_r][h_s] double.  Returns 0, or -1 when G is not positive
 * definite.
 */
int mfo_calib_solve(const double* gram, int h_s, int h_r, double ridge, double* W,
                    double* residual) {
  const int F = h_s + h_r;
  double* Lf = (double*)calloc((size_t)h_s * h_s, sizeof(double));
  for (int c = 0; c < h_s; ++c) {
    double d = gram[c * F + c] + ridge;
    for (int k = 0; k < c; ++k) d -= Lf[c * h_s + k] * Lf[c * h_s + k];
    if (!(d > 0.0)) { free(Lf); return -1; }
    Lf[c * h_s + c] = sqrt(d);
    for (int r = c + 1; r < h_s; ++r) {
      double v = gram[r * F + c];
      for (int k = 0; k < c; ++k) v -= Lf[r * h_s + k] * Lf[c * h_s + k];
      Lf[r * h_s + c] = v / Lf[c * h_s + c];
    }
  }
  double* z = (double*)malloc(sizeof(double) * (size_t)h_s);
  for (int r = 0; r < h_r; ++r) {
    /* forward: L z = c_r, backward: L^T w = z */
    for (int a = 0; a < h_s; ++a) {
      double v = gram[a * F + h_s + r];
      for (int k = 0; k < a; ++k) v -= Lf[a * h_s + k] * z[k];
      z[a] = v / Lf[a * h_s + a];
    }
    double* w = W + (int64_t)r * h_s;
    for (int a = h_s - 1; a >= 0; --a) {
      double v = z[a];
      for (int k = a + 1; k < h_s; ++k) v -= Lf[k * h_s + a] * w[k];
      w[a] = v / Lf[a * h_s + a];
    }
    if (residual) {
      double res = gram[(h_s + r) * F + h_s + r];
      for (int a = 0; a < h_s; ++a) {
        res -= 2.0 * w[a] * gram[a * F + h_s + r];
        for (int b = 0; b < h_s; ++b) res += w[a] * gram[a * F + b] * w[b];
      }
      residual[r] = res;
    }
  }
  free(z);
  free(Lf);
  return 0;
}

/*
 * Sender attention maps from the sender's own queries and keys, for compression without a
 * dense map (MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?", section
 * "存不下、读得慢?三个工程优化手段", subsection 1: block statistics first, then the kept
 * blocks, with no dense matrix assembled).  The map is the sender's causal attention
 * distribution:
 *   A_s[i][j] = exp(scale * <q_{i,s}, k_{j,g}>) / sum_{j' <= i} exp(scale * <q_{i,s}, k_{j',g}>)
 * for j <= i < L and 0 elsewhere, with g = floor(s * h_kv / h_s) (contiguous grouping of query
 * heads onto key heads).  The row maximum of the scaled products is subtracted before the
 * exponentials (the ratio is unchanged).  Q: [L][h_s][d], K: [L][h_kv][d] raw (dtype 0 f32,
 * 1 bf16); A: [h_s][Lp][Lp] double, fully written.
 */
static void qk_row(const void* Q, const void* K, int dtype, int h_s, int h_kv, int d, int s,
                   int i, double scale, double* z, double* out) {
  const int g = (int)((int64_t)s * h_kv / h_s);
  double zmax = -HUGE_VAL;
  for (int j = 0; j <= i; ++j) {
    double dot = 0.0;
    for (int c = 0; c < d; ++c)
      dot += value_at(Q, dtype, ((int64_t)i * h_s + s) * d + c) *
             value_at(K, dtype, ((int64_t)j * h_kv + g) * d + c);
    z[j] = scale * dot;
    if (z[j] > zmax) zmax = z[j];
  }
  double denom = 0.0;
  for (int j = 0; j <= i; ++j) denom += exp(z[j] - zmax);
  for (int j = 0; j <= i; ++j) out[j] = exp(z[j] - zmax) / denom;
}

void mfo_qk_maps(const void* Q, const void* K, int dtype, int L, int h_s, int h_kv, int d,
                 int64_t Lp, double scale, double* A) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  for (int64_t e = 0; e < (int64_t)h_s * Lp * Lp; ++e) A[e] = 0.0;
  for (int s = 0; s < h_s; ++s)
    for (int i = 0; i < L; ++i) qk_row(Q, K, dtype, h_s, h_kv, d, s, i, scale, z, A + ((int64_t)s * Lp + i) * Lp);
  free(z);
}

/* Rows [i0, i1) of the same maps (rows >= L are 0): out[s][i - i0][0 .. width), width >= i1. */
void mfo_qk_rows(const void* Q, const void* K, int dtype, int L, int h_s, int h_kv, int d,
                 int i0, int i1, int64_t width, double scale, double* out) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(i1 > 0 ? i1 : 1));
  for (int64_t e = 0; e < (int64_t)h_s * (i1 - i0) * width; ++e) out[e] = 0.0;
  for (int s = 0; s < h_s; ++s)
    for (int i = i0; i < i1 && i < L; ++i)
      qk_row(Q, K, dtype, h_s, h_kv, d, s, i, scale, z, out + ((int64_t)s * (i1 - i0) + (i - i0)) * width);
  free(z);
}
