/*
 * gdn_oracle.c -- plain, slow, single-threaded fp64 CPU oracle of the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file: only the
 * test suite, the smoke check and the CPU-baseline leg of the benchmark use it.  It shares no code,
 * header, table or constant with the CUDA library.
 *
 * What it computes.  The Ferrite project page (bhcc2025.github.io/ferrite), Design section 03
 * "Chunked Gated DeltaNet", names the method without writing it down: each linear-attention layer
 * carries a recurrent state for every request, a prompt is handled 32 rows at a time with the WY/UT
 * chunk form of the delta rule, its products on TF32 tensor cores (3xTF32 split), and the decoder
 * continues from the state the prompt leaves.  The page does not print the recurrence; the one used here is the published gated delta rule (Yang, Kautz and
 * Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta Rule", 2024/2025).  Per sequence
 * and head, with S_0 the initial state (dv x dk, zero when none is given):
 *
 *     S_t = alpha_t * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   alpha_t = exp(g_t)
 *     o_t = S_t q_t / sqrt(dk)
 *
 * q_t and k_t arrive already L2-normalised (the oracle never renormalises).
 *
 * Layouts (row-major, the same as the library's):
 *     q, k   [T_total, H, dk]      v, out  [T_total, H, dv]      g, beta  [T_total, H]
 *     state  [N, H, dv, dk]        cu_seqlens  int64[N + 1], cu[0] = 0, non-decreasing
 *
 * Functions
 *   gdn_oracle_recurrence  the recurrence token by token (the definition).  S(I - b k k^T) is
 *                          expanded as S - b (S k) k^T (associativity), nothing else is changed.
 *   gdn_oracle_rows        the same recurrence for chosen (sequence, head, row-of-S) triples only.
 *                          Right-multiplication acts on each row of S separately, so row r of S_t
 *                          needs only row r of S_{t-1}, k_t, q_t and the r-th entry of v_t.
 *   gdn_oracle_chunked     the chunkwise WY/UT evaluation of the same recurrence (Design section 03:
 *                          chunks of C rows, a unit-lower-triangular solve per chunk, W and U
 *                          matrices, intra-chunk attention, inter-chunk state carry) in fp64 for any
 *                          chunk size C >= 1.  It reaches the recurrence's result up to rounding.
 *
 * Every function returns 0 on success and a negative value on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX3(t, h, c, H, D) ((((int64_t)(t)) * (H) + (h)) * (D) + (c))

static int check_common(const int64_t* cu, int64_t n, int64_t H, int64_t dk, int64_t dv)
{
    if (!cu || n < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (cu[0] != 0) return -2;
    for (int64_t i = 0; i < n; ++i)
        if (cu[i + 1] < cu[i]) return -2;
    return 0;
}

int gdn_oracle_recurrence(const double* q, const double* k, const double* v, const double* g,
                          const double* beta, const int64_t* cu_seqlens, int64_t num_seqs,
                          const double* state_in, double* out, double* state_out, int64_t H,
                          int64_t dk, int64_t dv)
{
    int rc = check_common(cu_seqlens, num_seqs, H, dk, dv);
    if (rc) return rc;
    if (!q || !k || !v || !g || !beta || !out) return -1;
    const double scale = 1.0 / sqrt((double)dk);
    double* S = (double*)malloc(sizeof(double) * dv * dk);
    double* Sk = (double*)malloc(sizeof(double) * dv);
    if (!S || !Sk) { free(S); free(Sk); return -3; }

    for (int64_t n = 0; n < num_seqs; ++n) {
        for (int64_t h = 0; h < H; ++h) {
            /* S_0 */
            if (state_in)
                memcpy(S, state_in + ((n * H + h) * dv) * dk, sizeof(double) * dv * dk);
            else
                memset(S, 0, sizeof(double) * dv * dk);

            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                const double* kt = k + IDX3(t, h, 0, H, dk);
                const double* qt = q + IDX3(t, h, 0, H, dk);
                const double* vt = v + IDX3(t, h, 0, H, dv);
                const double a = exp(g[t * H + h]);
                const double b = beta[t * H + h];
                /* S_{t-1} k_t */
                for (int64_t r = 0; r < dv; ++r) {
                    double acc = 0.0;
                    for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * kt[c];
                    Sk[r] = acc;
                }
                /* S_t = a * (S - b (S k) k^T) + b v k^T */
                for (int64_t r = 0; r < dv; ++r)
                    for (int64_t c = 0; c < dk; ++c)
                        S[r * dk + c] = a * (S[r * dk + c] - b * Sk[r] * kt[c]) + b * vt[r] * kt[c];
                /* o_t = S_t q_t / sqrt(dk) */
                double* ot = out + IDX3(t, h, 0, H, dv);
                for (int64_t r = 0; r < dv; ++r) {
                    double acc = 0.0;
                    for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * qt[c];
                    ot[r] = acc * scale;
                }
            }
            if (state_out)
                memcpy(state_out + ((n * H + h) * dv) * dk, S, sizeof(double) * dv * dk);
        }
    }
    free(S);
    free(Sk);
    return 0;
}

/*
 * Sampled rows.  For sample i = (seq_idx[i], head_idx[i], row_idx[i]):
 *   out_rows[i * T_total + t] = o_t[h][r] for every t of that sequence (other entries untouched),
 *   state_rows[i * dk + c]    = S_L[r][c], the final state's row r.
 */
int gdn_oracle_rows(const double* q, const double* k, const double* v, const double* g,
                    const double* beta, const int64_t* cu_seqlens, int64_t num_seqs,
                    const double* state_in, int64_t H, int64_t dk, int64_t dv, int64_t n_samples,
                    const int64_t* seq_idx, const int64_t* head_idx, const int64_t* row_idx,
                    double* out_rows, double* state_rows)
{
    int rc = check_common(cu_seqlens, num_seqs, H, dk, dv);
    if (rc) return rc;
    if (!q || !k || !v || !g || !beta || !seq_idx || !head_idx || !row_idx) return -1;
    const int64_t T_total = cu_seqlens[num_seqs];
    const double scale = 1.0 / sqrt((double)dk);
    double* s = (double*)malloc(sizeof(double) * dk);
    if (!s) return -3;
    for (int64_t i = 0; i < n_samples; ++i) {
        const int64_t n = seq_idx[i], h = head_idx[i], r = row_idx[i];
        if (n < 0 || n >= num_seqs || h < 0 || h >= H || r < 0 || r >= dv) { free(s); return -1; }
        if (state_in)
            memcpy(s, state_in + (((n * H + h) * dv) + r) * dk, sizeof(double) * dk);
        else
            memset(s, 0, sizeof(double) * dk);
        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const double* kt = k + IDX3(t, h, 0, H, dk);
            const double* qt = q + IDX3(t, h, 0, H, dk);
            const double vr = v[IDX3(t, h, r, H, dv)];
            const double a = exp(g[t * H + h]);
            const double b = beta[t * H + h];
            double sk = 0.0;
            for (int64_t c = 0; c < dk; ++c) sk += s[c] * kt[c];
            for (int64_t c = 0; c < dk; ++c) s[c] = a * (s[c] - b * sk * kt[c]) + b * vr * kt[c];
            double o = 0.0;
            for (int64_t c = 0; c < dk; ++c) o += s[c] * qt[c];
            if (out_rows) out_rows[i * T_total + t] = o * scale;
        }
        if (state_rows) memcpy(state_rows + i * dk, s, sizeof(double) * dk);
    }
    free(s);
    return 0;
}

/*
 * Chunkwise WY/UT form, fp64, chunk size C.  Chunks restart at every sequence start; the last
 * chunk of a sequence may be shorter than C.  Inside a chunk of L rows (local index i = 0..L-1),
 * with S the state entering the chunk:
 *
 *   gamma_i = g_0 + ... + g_i                    (local cumulative log-gate)
 *   A_ij    = beta_i exp(gamma_i - gamma_j) (k_i . k_j)        for j < i, else 0
 *   T       = (I + A)^-1                          (forward substitution; unit lower triangular)
 *   W       = T diag(beta_j exp(gamma_j)) K      (L x dk)
 *   U'      = T diag(beta_j) V                    (L x dv)
 *   U       = U' - W S^T                          (the chunk's effective delta-rule writes)
 *   o_i     = scale * ( exp(gamma_i) S q_i + sum_{j<=i} exp(gamma_i - gamma_j) (q_i . k_j) U_j )
 *   S'      = exp(gamma_{L-1}) S + sum_j exp(gamma_{L-1} - gamma_j) U_j k_j^T
 *
 * Derivation: u_t = beta_t (v_t - alpha_t S_{t-1} k_t) turns the recurrence into
 * S_t = alpha_t S_{t-1} + u_t k_t^T; unrolling inside the chunk gives the triangular system
 * (I + A) U = diag(beta) V - diag(beta exp(gamma)) K S^T for the stacked u_t.
 */
int gdn_oracle_chunked(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, const int64_t* cu_seqlens, int64_t num_seqs,
                       const double* state_in, double* out, double* state_out, int64_t H,
                       int64_t dk, int64_t dv, int64_t C)
{
    int rc = check_common(cu_seqlens, num_seqs, H, dk, dv);
    if (rc) return rc;
    if (!q || !k || !v || !g || !beta || !out || C < 1) return -1;
    const double scale = 1.0 / sqrt((double)dk);
    double* S = (double*)malloc(sizeof(double) * dv * dk);
    double* Snew = (double*)malloc(sizeof(double) * dv * dk);
    double* gam = (double*)malloc(sizeof(double) * C);
    double* A = (double*)malloc(sizeof(double) * C * C);
    double* T = (double*)malloc(sizeof(double) * C * C);
    double* W = (double*)malloc(sizeof(double) * C * dk);
    double* U = (double*)malloc(sizeof(double) * C * dv);
    if (!S || !Snew || !gam || !A || !T || !W || !U) {
        free(S); free(Snew); free(gam); free(A); free(T); free(W); free(U);
        return -3;
    }

    for (int64_t n = 0; n < num_seqs; ++n) {
        for (int64_t h = 0; h < H; ++h) {
            if (state_in)
                memcpy(S, state_in + ((n * H + h) * dv) * dk, sizeof(double) * dv * dk);
            else
                memset(S, 0, sizeof(double) * dv * dk);

            for (int64_t t0 = cu_seqlens[n]; t0 < cu_seqlens[n + 1]; t0 += C) {
                int64_t L = cu_seqlens[n + 1] - t0;
                if (L > C) L = C;
#define KK(i, c) k[IDX3(t0 + (i), h, (c), H, dk)]
#define QQ(i, c) q[IDX3(t0 + (i), h, (c), H, dk)]
#define VV(i, r) v[IDX3(t0 + (i), h, (r), H, dv)]
#define GG(i) g[(t0 + (i)) * H + h]
#define BB(i) beta[(t0 + (i)) * H + h]
                /* local cumulative log-gate */
                double run = 0.0;
                for (int64_t i = 0; i < L; ++i) { run += GG(i); gam[i] = run; }
                /* A: strictly lower, beta- and decay-weighted key Gram matrix */
                for (int64_t i = 0; i < L; ++i)
                    for (int64_t j = 0; j < L; ++j) {
                        double a = 0.0;
                        if (j < i) {
                            double kk = 0.0;
                            for (int64_t c = 0; c < dk; ++c) kk += KK(i, c) * KK(j, c);
                            a = BB(i) * exp(gam[i] - gam[j]) * kk;
                        }
                        A[i * C + j] = a;
                    }
                /* T = (I + A)^-1 by forward substitution, row by row */
                for (int64_t i = 0; i < L; ++i)
                    for (int64_t j = 0; j < L; ++j) {
                        double t = (i == j) ? 1.0 : 0.0;
                        if (j < i) {
                            double acc = 0.0;
                            for (int64_t m = j; m < i; ++m) acc += A[i * C + m] * T[m * C + j];
                            t = -acc;
                        }
                        T[i * C + j] = t;
                    }
                /* W = T diag(beta exp(gamma)) K,  U = T diag(beta) V - W S^T */
                for (int64_t i = 0; i < L; ++i) {
                    for (int64_t c = 0; c < dk; ++c) {
                        double acc = 0.0;
                        for (int64_t j = 0; j <= i; ++j)
                            acc += T[i * C + j] * BB(j) * exp(gam[j]) * KK(j, c);
                        W[i * dk + c] = acc;
                    }
                    for (int64_t r = 0; r < dv; ++r) {
                        double acc = 0.0;
                        for (int64_t j = 0; j <= i; ++j) acc += T[i * C + j] * BB(j) * VV(j, r);
                        double ws = 0.0;
                        for (int64_t c = 0; c < dk; ++c) ws += W[i * dk + c] * S[r * dk + c];
                        U[i * dv + r] = acc - ws;
                    }
                }
                /* outputs: inter-chunk part through S, intra-chunk part through U */
                for (int64_t i = 0; i < L; ++i) {
                    double* oi = out + IDX3(t0 + i, h, 0, H, dv);
                    for (int64_t r = 0; r < dv; ++r) {
                        double inter = 0.0;
                        for (int64_t c = 0; c < dk; ++c) inter += S[r * dk + c] * QQ(i, c);
                        double intra = 0.0;
                        for (int64_t j = 0; j <= i; ++j) {
                            double qk = 0.0;
                            for (int64_t c = 0; c < dk; ++c) qk += QQ(i, c) * KK(j, c);
                            intra += exp(gam[i] - gam[j]) * qk * U[j * dv + r];
                        }
                        oi[r] = scale * (exp(gam[i]) * inter + intra);
                    }
                }
                /* state carry */
                const double gl = gam[L - 1];
                for (int64_t r = 0; r < dv; ++r)
                    for (int64_t c = 0; c < dk; ++c) {
                        double acc = exp(gl) * S[r * dk + c];
                        for (int64_t j = 0; j < L; ++j)
                            acc += exp(gl - gam[j]) * U[j * dv + r] * KK(j, c);
                        Snew[r * dk + c] = acc;
                    }
                memcpy(S, Snew, sizeof(double) * dv * dk);
#undef KK
#undef QQ
#undef VV
#undef GG
#undef BB
            }
            if (state_out)
                memcpy(state_out + ((n * H + h) * dv) * dk, S, sizeof(double) * dv * dk);
        }
    }
    free(S); free(Snew); free(gam); free(A); free(T); free(W); free(U);
    return 0;
}
