/*
 * CPU oracle for the RotateAttention INT4 attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, independent
 * definition that the CUDA path is checked against.  Only the tests, the
 * package's smoke() check and bench.py's CPU-baseline leg may load it; the
 * product path never does.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Source: "RotateAttention: RoPE-Aware Rotation and Range Rectification for
 * INT4 Quantized Attention in Video Generation" (arXiv 2607.02584), as
 * described on the papernotes.org page (sections "overall framework" and
 * "key design 1-3"), the gecl reading notes ("Method") and the abstract.
 *
 * Precision rules.  Wherever a floating-point value decides an integer code
 * (the Q/K/V INT4 codes, the P codes) the computation is carried out in fp32
 * with the operation order spelled out below and no contraction (build with
 * -ffp-contract=off), because that is the precision the CUDA path decides in.
 * Everything else (channel means, the attention accumulators, the reference
 * attention) is fp64.
 *
 * Readings of points the pages leave open:
 *   R1 RoPE pairs are adjacent channels (2k, 2k+1) of a segment; the segment's
 *      frequencies are theta^(-2k/Dj); rotation by angle p*freq is the complex
 *      product (x0 + i x1) e^{i phi}.
 *   R2 RoPE is applied first, then the orthogonal rotation R (row vectors:
 *      x M R); H2 = [[1,1],[1,-1]]/sqrt(2).
 *   R3 K smoothing subtracts the per-channel mean over all N tokens of the
 *      rotated K; Q is not smoothed.  The mean is taken as R applied (in fp64)
 *      to the fp64 mean of the RoPE'd K, which equals the mean of the rotated
 *      K because R is linear and the same for every token; rounded once to
 *      fp32.
 *   R4 Q and K: per-token symmetric INT4, scale s = amax/7 (fp32), code =
 *      clamp(rint(x * inv), -7, 7) with inv = fl(7/amax) and the product
 *      x * inv taken exactly (one rounding, in the rint, ties to even);
 *      amax = 0 gives s = 0 and codes 0.
 *   R5 V: per-channel symmetric INT4 over all N tokens, same rule.
 *   R6 P codes use the running row maximum after the current key block:
 *      c = clamp(rint(15 * exp(S - m)), 0, 15) - 8.
 *   R7 The softmax denominator is the sum of the dequantised P codes,
 *      sum (c + 8) / 15, with the same online rescaling as the numerator.
 *   R8 Keys past N in the last block do not take part (S = -inf, code -8,
 *      V = 0, excluded from colsum).
 *   R9 S = ((float)S_int * s_k[j]) * (s_q[i] * (1/sqrt(D))) in fp32.
 *   R11 Ablation switches (off by default): p_mode LOCAL takes the codes of
 *      a block against that block's own maximum and weights the block by
 *      exp(m_block - m) in the recurrence; p_mode SYMMETRIC uses the
 *      SageAttention-style codes c = rint(7 exp(S - m)) in [0, 7] with no zero
 *      point, dequantised as c / 7; l_mode FP32 makes the denominator the
 *      plain sum of exp(S - m_codes) instead of the dequantised code sum.
 *   R12 The full rotation (rot 3) is RoPE followed by the row times H_D /
 *      sqrt(D), H_D the Sylvester Hadamard matrix, evaluated as butterflies
 *      at distances 1, 2, ..., D/2 in fp32 and one final scaling.
 *   R10 Codes are packed two per byte, element 2t in the low nibble, as
 *      4-bit two's complement.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int B, H, N, D;
  int seg[3];     /* frame / height / width channel counts, sum = D */
  int grid[3];    /* frame / height / width extents of the token grid */
  double theta;   /* RoPE base */
  int rot;        /* 0 = RoPE only, 1 = interleaved, 2 = half, 3 = full Hadamard rotation */
  int block_q, block_k;
  int p_mode;     /* ORC_P_RANGE (default), ORC_P_LOCAL, ORC_P_SYMMETRIC (R11) */
  int l_mode;     /* ORC_L_CODES (default), ORC_L_FP32 (R11) */
} orc_problem;

enum { ORC_OK = 0, ORC_BAD = 1 };
enum { ORC_P_RANGE = 0, ORC_P_LOCAL = 1, ORC_P_SYMMETRIC = 2 };
enum { ORC_L_CODES = 0, ORC_L_FP32 = 1 };

static int seg_off(const orc_problem* p, int j) {
  int o = 0;
  for (int i = 0; i < j; ++i) o += p->seg[i];
  return o;
}

static int check_problem(const orc_problem* p) {
  if (p->B < 1 || p->H < 1 || p->N < 1 || p->D < 2 || p->D > 256) return ORC_BAD;
  if (p->seg[0] + p->seg[1] + p->seg[2] != p->D) return ORC_BAD;
  for (int j = 0; j < 3; ++j) {
    if (p->seg[j] < 2 || p->seg[j] % 2) return ORC_BAD;
    if (p->grid[j] < 1) return ORC_BAD;
  }
  if (p->grid[0] * p->grid[1] * p->grid[2] < 1) return ORC_BAD;
  if (p->rot < 0 || p->rot > 3 || p->block_k < 1) return ORC_BAD;
  if (p->rot == 3 && (p->D & (p->D - 1))) return ORC_BAD;  /* Sylvester H_D needs D = 2^k */
  if (p->p_mode < ORC_P_RANGE || p->p_mode > ORC_P_SYMMETRIC) return ORC_BAD;
  if (p->l_mode < ORC_L_CODES || p->l_mode > ORC_L_FP32) return ORC_BAD;
  return ORC_OK;
}

/* Number of table entries (pairs x positions summed over segments). */
int orc_table_len(const orc_problem* p) {
  int n = 0;
  for (int j = 0; j < 3; ++j) n += p->grid[j] * (p->seg[j] / 2);
  return n;
}

/*
 * RoPE tables (papernotes page, key design 1: D = Df + Dh + Dw, the 3D RoPE
 * matrix M is block-diagonal in 2x2 rotation blocks; interleaved rotation
 * pre-multiplies H2 into those blocks, "M' = RM", stored as static parameters).
 * Angles and entries are computed in fp64 and rounded once to fp32.
 * Entry (segment j, position g, pair k) sits at off_j + g * (Dj/2) + k.
 *   rot 0 / 2: a = cos(phi), b = sin(phi)
 *   rot 1    : a = (cos + sin)/sqrt2, b = (cos - sin)/sqrt2, so that the fused
 *              2x2 block is [[a, b], [b, -a]] acting on row vectors.
 */
int orc_rope_tables(const orc_problem* p, float* tab_a, float* tab_b) {
  if (check_problem(p)) return ORC_BAD;
  int base = 0;
  for (int j = 0; j < 3; ++j) {
    int dj = p->seg[j], npair = dj / 2;
    for (int g = 0; g < p->grid[j]; ++g) {
      for (int k = 0; k < npair; ++k) {
        double freq = pow(p->theta, -2.0 * (double)k / (double)dj);
        double phi = (double)g * freq;
        double c = cos(phi), s = sin(phi);
        int idx = base + g * npair + k;
        if (p->rot == 1) {
          tab_a[idx] = (float)((c + s) / sqrt(2.0));
          tab_b[idx] = (float)((c - s) / sqrt(2.0));
        } else {
          tab_a[idx] = (float)c;
          tab_b[idx] = (float)s;
        }
      }
    }
    base += p->grid[j] * npair;
  }
  return ORC_OK;
}

/*
 * RoPE + RoPE-aware rotation of one token row (papernotes page, key design 1;
 * gecl notes, "Method").  fp32, operation order as written, no contraction.
 *   interleaved: out0 = x0*a + x1*b ; out1 = x0*b - x1*a   (fused table)
 *   half       : r0 = x0*c - x1*s ; r1 = x0*s + x1*c      (RoPE)
 *                then per segment, h = Dj/2, i < h:
 *                out[2i] = (r_i + r_{i+h}) * (1/sqrt2), out[2i+1] = (r_i - r_{i+h}) * (1/sqrt2)
 *   none       : RoPE only.
 *   full       : RoPE (as half), then the whole row times H_D / sqrt(D), H_D
 *                the Sylvester Hadamard matrix (the full D x D rotation of the
 *                pages' ablation): butterflies (a, b) -> (a + b, a - b) on
 *                channel pairs d apart for d = 1, 2, 4, ..., D/2 in that
 *                order, then one multiplication by fp32(1/sqrt(D)).
 * swap_order != 0 applies the half-rotation before RoPE instead (used only by a
 * test that shows the other order breaks QK^T invariance).
 */
static void rope_rotate_row(const orc_problem* p, const float* ta, const float* tb,
                            const int32_t* pos3, const float* x, float* out, int swap_order) {
  float tmp[256];
  const float r2 = (float)(1.0 / sqrt(2.0));
  int base = 0;
  for (int j = 0; j < 3; ++j) {
    int o = seg_off(p, j), dj = p->seg[j], npair = dj / 2;
    int g = pos3[j];
    const float* src = x + o;
    float pre[256];
    if (swap_order && p->rot == 2) {
      for (int i = 0; i < npair; ++i) {
        float u = src[i], w = src[i + npair];
        pre[2 * i] = (u + w) * r2;
        pre[2 * i + 1] = (u - w) * r2;
      }
      src = pre;
    }
    for (int k = 0; k < npair; ++k) {
      float a = ta[base + g * npair + k], b = tb[base + g * npair + k];
      float x0 = src[2 * k], x1 = src[2 * k + 1];
      float y0, y1;
      if (p->rot == 1) {
        y0 = x0 * a + x1 * b;
        y1 = x0 * b - x1 * a;
      } else {
        y0 = x0 * a - x1 * b;
        y1 = x0 * b + x1 * a;
      }
      tmp[o + 2 * k] = y0;
      tmp[o + 2 * k + 1] = y1;
    }
    if (p->rot == 2 && !swap_order) {
      for (int i = 0; i < npair; ++i) {
        float u = tmp[o + i], w = tmp[o + i + npair];
        out[o + 2 * i] = (u + w) * r2;
        out[o + 2 * i + 1] = (u - w) * r2;
      }
    } else {
      for (int d = 0; d < dj; ++d) out[o + d] = tmp[o + d];
    }
    base += p->grid[j] * npair;
  }
  if (p->rot == 3) {
    const int D = p->D;
    for (int d = 1; d < D; d <<= 1)
      for (int i = 0; i < D; ++i)
        if (!(i & d)) {
          float a = out[i], b = out[i + d];
          out[i] = a + b;
          out[i + d] = a - b;
        }
    const float c = (float)(1.0 / sqrt((double)D));
    for (int i = 0; i < D; ++i) out[i] = out[i] * c;
  }
}

int orc_rope_rotate(const orc_problem* p, const float* x, const int32_t* pos,
                    float* out, int swap_order) {
  if (check_problem(p)) return ORC_BAD;
  int tl = orc_table_len(p);
  float* ta = (float*)malloc(sizeof(float) * tl);
  float* tb = (float*)malloc(sizeof(float) * tl);
  orc_rope_tables(p, ta, tb);
  for (int n = 0; n < p->N; ++n) {
    for (int j = 0; j < 3; ++j)
      if (pos[3 * n + j] < 0 || pos[3 * n + j] >= p->grid[j]) { free(ta); free(tb); return ORC_BAD; }
    rope_rotate_row(p, ta, tb, pos + 3 * n, x + (size_t)n * p->D, out + (size_t)n * p->D, swap_order);
  }
  free(ta);
  free(tb);
  return ORC_OK;
}

/* The rotation R of rope_rotate_row applied to a D-vector in fp64 (no RoPE):
 * interleaved: (m_2k +- m_2k+1)/sqrt2 on adjacent pairs; half: per segment
 * (m_i +- m_i+h)/sqrt2 to positions 2i, 2i+1; full: m H_D / sqrt(D)
 * (Sylvester, entry (-1)^popcount(e & d)); none: m. */
static void rotate_mean(const orc_problem* p, const double* m, double* out) {
  const int D = p->D;
  const double r2 = 1.0 / sqrt(2.0);
  if (p->rot == 1) {
    for (int d = 0; d < D; d += 2) {
      out[d] = (m[d] + m[d + 1]) * r2;
      out[d + 1] = (m[d] - m[d + 1]) * r2;
    }
  } else if (p->rot == 2) {
    int o = 0;
    for (int j = 0; j < 3; ++j) {
      const int h = p->seg[j] / 2;
      for (int i = 0; i < h; ++i) {
        out[o + 2 * i] = (m[o + i] + m[o + i + h]) * r2;
        out[o + 2 * i + 1] = (m[o + i] - m[o + i + h]) * r2;
      }
      o += p->seg[j];
    }
  } else if (p->rot == 3) {
    const double c = 1.0 / sqrt((double)D);
    for (int d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int e = 0; e < D; ++e) acc += (__builtin_popcount((unsigned)(e & d)) & 1) ? -m[e] : m[e];
      out[d] = acc * c;
    }
  } else {
    for (int d = 0; d < D; ++d) out[d] = m[d];
  }
}

/* Symmetric INT4 code of x given the reciprocal inv = fl(7/amax) (reading
 * R4/R5): rint, ties to even, of the exact product x * inv (two fp32 values:
 * their product is exact in fp64). */
static int quant4(float x, float inv) {
  double y = (double)x * (double)inv;
  double r = rint(y);
  if (r > 7.0) r = 7.0;
  if (r < -7.0) r = -7.0;
  return (int)r;
}

static void pack_row(const int* codes, int D, uint8_t* dst) {
  for (int t = 0; t < D / 2; ++t)
    dst[t] = (uint8_t)((codes[2 * t] & 0xF) | ((codes[2 * t + 1] & 0xF) << 4));
}

/* Per-token INT4 of one row (gecl notes, "Key Insight": per-token INT4 for Q and K). */
static void quant_token(const float* x, int D, uint8_t* dst, float* scale) {
  float amax = 0.0f;
  for (int d = 0; d < D; ++d) {
    float a = fabsf(x[d]);
    if (a > amax) amax = a;
  }
  int codes[256];
  if (amax == 0.0f) {
    *scale = 0.0f;
    for (int d = 0; d < D; ++d) codes[d] = 0;
  } else {
    float inv = 7.0f / amax;
    *scale = amax / 7.0f;
    for (int d = 0; d < D; ++d) codes[d] = quant4(x[d], inv);
  }
  pack_row(codes, D, dst);
}

/*
 * Prologue for one (b, h) head: RoPE + rotation of Q and K, K smoothing,
 * per-token INT4 of Q and K, per-channel INT4 of V and per-block V column sums.
 * papernotes page, "overall framework" (smoothing, rotation, quantised V) and
 * key design 1; gecl notes "Method".  Inputs q, k, v are [N, D] fp32.
 * Outputs: q4/k4/v4 [N, D/2] packed, sq/sk [N], kmean/sv [D],
 * colsum [ceil(N/block_k), D].  k_rot (nullable) receives K after RoPE +
 * rotation and before smoothing; q_rot (nullable) receives Q after RoPE +
 * rotation.
 */
int orc_prologue_head(const orc_problem* p, const float* q, const float* k, const float* v,
                      const int32_t* pos, uint8_t* q4, float* sq, uint8_t* k4, float* sk,
                      float* kmean, uint8_t* v4, float* sv, int32_t* colsum,
                      float* q_rot, float* k_rot) {
  if (check_problem(p)) return ORC_BAD;
  const int N = p->N, D = p->D;
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < 3; ++j)
      if (pos[3 * n + j] < 0 || pos[3 * n + j] >= p->grid[j]) return ORC_BAD;
  int tl = orc_table_len(p);
  float* ta = (float*)malloc(sizeof(float) * tl);
  float* tb = (float*)malloc(sizeof(float) * tl);
  float* kr = (float*)malloc(sizeof(float) * (size_t)N * D);
  orc_rope_tables(p, ta, tb);

  /* Q: rotate, per-token quantise. */
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    float row[256];
    rope_rotate_row(p, ta, tb, pos + 3 * n, q + (size_t)n * D, row, 0);
    if (q_rot) memcpy(q_rot + (size_t)n * D, row, sizeof(float) * D);
    quant_token(row, D, q4 + (size_t)n * (D / 2), sq + n);
  }
  /* K: rotate. */
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    rope_rotate_row(p, ta, tb, pos + 3 * n, k + (size_t)n * D, kr + (size_t)n * D, 0);
  if (k_rot) memcpy(k_rot, kr, sizeof(float) * (size_t)N * D);
  /* K channel mean over all tokens of the rotated K (reading R3): the rotation
   * R is linear and the same for every token, so mean(x M_n R) = mean(x M_n) R.
   * The mean of the RoPE'd K (no rotation) is summed in fp64, R is applied to
   * that D-vector in fp64, and the result is rounded once to fp32. */
  {
    orc_problem p0 = *p;
    p0.rot = 0;
    float* ta0 = (float*)malloc(sizeof(float) * tl);
    float* tb0 = (float*)malloc(sizeof(float) * tl);
    orc_rope_tables(&p0, ta0, tb0);
    double m[256], mr[256];
    for (int d = 0; d < D; ++d) m[d] = 0.0;
    for (int n = 0; n < N; ++n) {
      float row[256];
      rope_rotate_row(&p0, ta0, tb0, pos + 3 * n, k + (size_t)n * D, row, 0);
      for (int d = 0; d < D; ++d) m[d] += (double)row[d];
    }
    for (int d = 0; d < D; ++d) m[d] /= (double)N;
    rotate_mean(p, m, mr);
    for (int d = 0; d < D; ++d) kmean[d] = (float)mr[d];
    free(ta0);
    free(tb0);
  }
  /* K: smooth, per-token quantise. */
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    float row[256];
    for (int d = 0; d < D; ++d) row[d] = kr[(size_t)n * D + d] - kmean[d];
    quant_token(row, D, k4 + (size_t)n * (D / 2), sk + n);
  }
  /* V: per-channel scale over all tokens, codes, per-block column sums. */
  float inv[256];
  for (int d = 0; d < D; ++d) {
    float amax = 0.0f;
    for (int n = 0; n < N; ++n) {
      float a = fabsf(v[(size_t)n * D + d]);
      if (a > amax) amax = a;
    }
    sv[d] = amax / 7.0f;
    inv[d] = amax == 0.0f ? 0.0f : 7.0f / amax;
  }
  int nb = (N + p->block_k - 1) / p->block_k;
  memset(colsum, 0, sizeof(int32_t) * (size_t)nb * D);
  for (int n = 0; n < N; ++n) {
    int codes[256];
    for (int d = 0; d < D; ++d) {
      codes[d] = inv[d] == 0.0f ? 0 : quant4(v[(size_t)n * D + d], inv[d]);
      colsum[(size_t)(n / p->block_k) * D + d] += codes[d];
    }
    pack_row(codes, D, v4 + (size_t)n * (D / 2));
  }
  free(ta);
  free(tb);
  free(kr);
  return ORC_OK;
}

static int unpack4(const uint8_t* row, int d) {
  int nib = (row[d >> 1] >> ((d & 1) * 4)) & 0xF;
  return nib >= 8 ? nib - 16 : nib;
}

/*
 * Range-rectified P code (papernotes page, key design 2): with P = exp(S - m)
 * in (0, 1] and the fixed scale 15 and zero point -8, c = round(15 P) - 8 in
 * [-8, 7].  S and m are the fp32 values; exp, the product and rint are
 * evaluated in fp64 (ties to even).
 */
int orc_p_code(float S, float m) {
  if (isinf(S) && S < 0) return -8;
  double e = exp((double)S - (double)m);
  double r = rint(15.0 * e);
  if (r < 0.0) r = 0.0;
  if (r > 15.0) r = 15.0;
  return (int)r - 8;
}

/*
 * Symmetric P code of the SageAttention-style baseline that the pages compare
 * against (papernotes page, key design 2: only the levels 0..7 of the signed
 * range are used): c = round(7 P) in [0, 7], P = exp(S - m), no zero point.
 * Same precision rules as orc_p_code.
 */
int orc_p_code_sym(float S, float m) {
  if (isinf(S) && S < 0) return 0;
  double e = exp((double)S - (double)m);
  double r = rint(7.0 * e);
  if (r < 0.0) r = 0.0;
  if (r > 7.0) r = 7.0;
  return (int)r;
}

/*
 * Blocked attention of rows [row0, row1) of one head with online softmax
 * (papernotes page: "overall framework" flowchart D-F, key design 2; the
 * FlashAttention recurrence with the running ("sliding") row maximum).
 *
 * quant != 0: the INT4 path.  S from codes (reading R9), P codes from
 *   orc_p_code against the running max m_t after block t (R6),
 *   acc_t[d] = sum_j c_ij v4_jd + 8 colsum_t[d] (the zero-point correction),
 *   O <- alpha O + (s_v/15) acc_t, l <- alpha l + lq_t/15 (R7).
 *   With the R11 switches: the codes are taken against m_c (the block's own
 *   maximum for LOCAL, else m_t) and the block enters with the weight
 *   beta = exp(m_c - m_t); SYMMETRIC codes have 7 levels and no zero point
 *   (acc_t = sum_j c_ij v4_jd, scale s_v/7, lq_t/7); FP32 replaces lq_t/L by
 *   sum_j exp(S_ij - m_c).
 * quant == 0: the same recurrence on fp64 inputs qf/kf/vf with
 *   S = q.k / sqrt(D) and P = exp(S - m) (no quantisation) -- used by the
 *   tests to show that the blocked recurrence equals plain softmax attention.
 *
 * out: [row1-row0, D] fp64 (O / l).  lse (nullable): m + ln(l).
 * Dumps (nullable; quant only): s_dump [rows, N] S_int, c_dump [rows, N] codes,
 * acc_dump [rows, nblocks, D] per-block acc_t.
 */
typedef struct {
  const uint8_t *q4, *k4, *v4;
  const float *sq, *sk, *sv;
  const int32_t* colsum;
  const double *qf, *kf, *vf;
  const int8_t* codes_in;  /* nullable [rows, N]: P codes to use instead of computing them */
  int row0;
} orc_attn_in;

static void attn_row(const orc_problem* p, const orc_attn_in* in, int quant, int i,
                     double* out, double* lse, int32_t* s_dump, int8_t* c_dump,
                     int32_t* acc_dump) {
  const int N = p->N, D = p->D, Bk = p->block_k;
  const int nb = (N + Bk - 1) / Bk;
  const float inv_sqrt_d = (float)(1.0 / sqrt((double)D));
  double O[256], acc[256];
  double l = 0.0;
  float m = -INFINITY;          /* quant: fp32 running max of fp32 S */
  double md = -INFINITY;        /* exact mode running max */
  int qi[256];
  float ci = 0.0f;
  if (quant) {
    for (int d = 0; d < D; ++d) qi[d] = unpack4(in->q4 + (size_t)i * (D / 2), d);
    ci = in->sq[i] * inv_sqrt_d;
  }
  for (int d = 0; d < D; ++d) O[d] = 0.0;
  float* S = (float*)malloc(sizeof(float) * Bk);
  double* Sd = (double*)malloc(sizeof(double) * Bk);
  for (int t = 0; t < nb; ++t) {
    int j0 = t * Bk, j1 = j0 + Bk < N ? j0 + Bk : N;
    double alpha;
    if (quant) {
      float mt = m, mb = -INFINITY;
      for (int j = j0; j < j1; ++j) {
        const uint8_t* kr = in->k4 + (size_t)j * (D / 2);
        int32_t sint = 0;
        for (int d = 0; d < D; ++d) sint += qi[d] * unpack4(kr, d);
        if (s_dump) s_dump[j] = sint;
        float v = (float)sint * in->sk[j];
        S[j - j0] = v * ci;
        if (S[j - j0] > mt) mt = S[j - j0];
        if (S[j - j0] > mb) mb = S[j - j0];
      }
      alpha = (m == -INFINITY) ? 0.0 : exp((double)m - (double)mt);
      m = mt;
      const int sym = p->p_mode == ORC_P_SYMMETRIC;
      const float mc = p->p_mode == ORC_P_LOCAL ? mb : m;   /* the max the codes use */
      const double beta = exp((double)mc - (double)m);      /* 1 unless LOCAL */
      const int zp = sym ? 0 : 8;
      const double levels = sym ? 7.0 : 15.0;
      int lq = 0;
      double le = 0.0;
      for (int d = 0; d < D; ++d) acc[d] = 0.0;
      int32_t acci[256];
      for (int d = 0; d < D; ++d) acci[d] = 0;
      for (int j = j0; j < j1; ++j) {
        int c = in->codes_in ? in->codes_in[(size_t)(i - in->row0) * N + j]
                             : (sym ? orc_p_code_sym(S[j - j0], mc) : orc_p_code(S[j - j0], mc));
        if (c_dump) c_dump[j] = (int8_t)c;
        lq += c + zp;
        le += exp((double)S[j - j0] - (double)mc);
        const uint8_t* vr = in->v4 + (size_t)j * (D / 2);
        for (int d = 0; d < D; ++d) acci[d] += c * unpack4(vr, d);
      }
      for (int d = 0; d < D; ++d) {
        acci[d] += zp * in->colsum[(size_t)t * D + d];
        if (acc_dump) acc_dump[(size_t)t * D + d] = acci[d];
        acc[d] = (double)in->sv[d] / levels * (double)acci[d];
      }
      for (int d = 0; d < D; ++d) O[d] = alpha * O[d] + beta * acc[d];
      l = alpha * l + beta * (p->l_mode == ORC_L_FP32 ? le : (double)lq / levels);
    } else {
      double mt = md;
      for (int j = j0; j < j1; ++j) {
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += in->qf[(size_t)i * D + d] * in->kf[(size_t)j * D + d];
        Sd[j - j0] = s / sqrt((double)D);
        if (Sd[j - j0] > mt) mt = Sd[j - j0];
      }
      alpha = (md == -INFINITY) ? 0.0 : exp(md - mt);
      md = mt;
      double lt = 0.0;
      for (int d = 0; d < D; ++d) acc[d] = 0.0;
      for (int j = j0; j < j1; ++j) {
        double pj = exp(Sd[j - j0] - md);
        lt += pj;
        for (int d = 0; d < D; ++d) acc[d] += pj * in->vf[(size_t)j * D + d];
      }
      for (int d = 0; d < D; ++d) O[d] = alpha * O[d] + acc[d];
      l = alpha * l + lt;
    }
  }
  for (int d = 0; d < D; ++d) out[d] = O[d] / l;
  if (lse) *lse = (quant ? (double)m : md) + log(l);
  free(S);
  free(Sd);
}

static void attn_rows(const orc_problem* p, const orc_attn_in* in, int quant, int row0, int row1,
                      double* out, double* lse, int32_t* s_dump, int8_t* c_dump, int32_t* acc_dump) {
  const int N = p->N, D = p->D;
  const int nb = (N + p->block_k - 1) / p->block_k;
#pragma omp parallel for schedule(dynamic, 4)
  for (int i = row0; i < row1; ++i) {
    size_t r = (size_t)(i - row0);
    attn_row(p, in, quant, i, out + r * D, lse ? lse + r : NULL,
             s_dump ? s_dump + r * N : NULL, c_dump ? c_dump + r * N : NULL,
             acc_dump ? acc_dump + r * (size_t)nb * D : NULL);
  }
}

int orc_attention_int4_rows(const orc_problem* p, const uint8_t* q4, const float* sq,
                            const uint8_t* k4, const float* sk, const uint8_t* v4,
                            const float* sv, const int32_t* colsum, int row0, int row1,
                            double* out, double* lse, int32_t* s_dump, int8_t* c_dump,
                            int32_t* acc_dump) {
  if (check_problem(p) || row0 < 0 || row1 > p->N || row0 >= row1) return ORC_BAD;
  orc_attn_in in = {q4, k4, v4, sq, sk, sv, colsum, NULL, NULL, NULL, NULL, row0};
  attn_rows(p, &in, 1, row0, row1, out, lse, s_dump, c_dump, acc_dump);
  return ORC_OK;
}

/*
 * The same INT4 attention with the P codes supplied by the caller
 * (codes_in [row1-row0, N], values in [-8, 7]) instead of computed: the
 * running maximum, the online rescaling and the accumulation are unchanged.
 * Used to check an implementation's accumulation on its own codes.
 */
int orc_attention_int4_rows_given_codes(const orc_problem* p, const uint8_t* q4, const float* sq,
                                        const uint8_t* k4, const float* sk, const uint8_t* v4,
                                        const float* sv, const int32_t* colsum, const int8_t* codes_in,
                                        int row0, int row1, double* out, double* lse) {
  if (check_problem(p) || row0 < 0 || row1 > p->N || row0 >= row1 || !codes_in) return ORC_BAD;
  for (size_t i = 0; i < (size_t)(row1 - row0) * p->N; ++i)
    if (codes_in[i] < -8 || codes_in[i] > 7) return ORC_BAD;
  orc_attn_in in = {q4, k4, v4, sq, sk, sv, colsum, NULL, NULL, NULL, codes_in, row0};
  attn_rows(p, &in, 1, row0, row1, out, lse, NULL, NULL, NULL);
  return ORC_OK;
}

int orc_attention_exact_blocked_rows(const orc_problem* p, const double* q, const double* k,
                                     const double* v, int row0, int row1, double* out,
                                     double* lse) {
  if (check_problem(p) || row0 < 0 || row1 > p->N || row0 >= row1) return ORC_BAD;
  orc_attn_in in = {NULL, NULL, NULL, NULL, NULL, NULL, NULL, q, k, v, NULL, row0};
  attn_rows(p, &in, 0, row0, row1, out, lse, NULL, NULL, NULL);
  return ORC_OK;
}

/* ---- explicit fp64 matrices, for the invariance tests ------------------ */

/*
 * The orthogonal rotation R (D x D, row-vector convention x -> x R), built from
 * the definitions on the papernotes page, key design 1:
 *   interleaved: block-diagonal of D/2 copies of H2 on channel pairs (2i, 2i+1);
 *   half: per segment, a permutation placing channel i and i + Dj/2 at 2i, 2i+1,
 *         followed by Dj/2 copies of H2 on those adjacent pairs;
 *   none: the identity;
 *   full: the normalised Sylvester Hadamard matrix H_D / sqrt(D).
 */
int orc_rotation_matrix(const orc_problem* p, double* R) {
  if (check_problem(p)) return ORC_BAD;
  const int D = p->D;
  const double r2 = 1.0 / sqrt(2.0);
  memset(R, 0, sizeof(double) * D * D);
  if (p->rot == 0) {
    for (int d = 0; d < D; ++d) R[d * D + d] = 1.0;
    return ORC_OK;
  }
  if (p->rot == 3) {  /* H_D / sqrt(D), H_D[i][j] = (-1)^popcount(i & j) */
    for (int i = 0; i < D; ++i)
      for (int j = 0; j < D; ++j) {
        int b = i & j, par = 0;
        while (b) { par ^= b & 1; b >>= 1; }
        R[i * D + j] = (par ? -1.0 : 1.0) / sqrt((double)D);
      }
    return ORC_OK;
  }
  double* Pi = (double*)calloc((size_t)D * D, sizeof(double));
  double* Hb = (double*)calloc((size_t)D * D, sizeof(double));
  for (int j = 0; j < 3; ++j) {
    int o = seg_off(p, j), h = p->seg[j] / 2;
    for (int i = 0; i < h; ++i) {
      if (p->rot == 2) {
        Pi[(o + i) * D + (o + 2 * i)] = 1.0;
        Pi[(o + i + h) * D + (o + 2 * i + 1)] = 1.0;
      } else {
        Pi[(o + 2 * i) * D + (o + 2 * i)] = 1.0;
        Pi[(o + 2 * i + 1) * D + (o + 2 * i + 1)] = 1.0;
      }
      int a = o + 2 * i, b = a + 1;
      Hb[a * D + a] = r2;
      Hb[a * D + b] = r2;
      Hb[b * D + a] = r2;
      Hb[b * D + b] = -r2;
    }
  }
  for (int r = 0; r < D; ++r)
    for (int c = 0; c < D; ++c) {
      double s = 0.0;
      for (int t = 0; t < D; ++t) s += Pi[r * D + t] * Hb[t * D + c];
      R[r * D + c] = s;
    }
  free(Pi);
  free(Hb);
  return ORC_OK;
}

/*
 * The 3D RoPE matrix M_n (D x D, row vectors) of a token at grid position pos3,
 * in fp64 with exact cos/sin: 2x2 blocks [[c, s], [-s, c]] on channel pairs
 * (o_j + 2k, o_j + 2k + 1), angle pos3[j] * theta^(-2k/Dj).
 */
int orc_rope_matrix(const orc_problem* p, const int32_t* pos3, double* M) {
  if (check_problem(p)) return ORC_BAD;
  const int D = p->D;
  memset(M, 0, sizeof(double) * D * D);
  for (int j = 0; j < 3; ++j) {
    int o = seg_off(p, j), dj = p->seg[j];
    for (int k = 0; k < dj / 2; ++k) {
      double phi = (double)pos3[j] * pow(p->theta, -2.0 * (double)k / (double)dj);
      double c = cos(phi), s = sin(phi);
      int a = o + 2 * k, b = a + 1;
      M[a * D + a] = c;
      M[a * D + b] = s;
      M[b * D + a] = -s;
      M[b * D + b] = c;
    }
  }
  return ORC_OK;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
