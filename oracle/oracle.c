/*
 * oracle.c -- plain, slow, fp64 CPU oracle for paged sparse-attention prefill
 * with query unions.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the bench's CPU-baseline leg call it; the product path never does.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (PageWeaver: KV-Guided Query Unions for Sparse Attention,
 * Abstract and Figure 1): every query keeps exactly its own TopK page support
 * and owns its output row.  For Q head h' (KV head h = h' / g) and query i at
 * position p_i:
 *
 *   A_i  = { t = u*T + o : u in set(topk[h'][i][:]) minus {-1}, 0 <= o < T,
 *            t < kv_len, t <= p_i }                 (causal inside a page)
 *   s_t  = softmax_scale * sum_d q[i][h'][d] * k[t][h][d]
 *   O    = sum_{t in A_i} softmax(s)_t * v[t][h]
 *
 * evaluated two-pass in fp64 (max, then the exponential sum and the weighted
 * sum).  Token t lives in logical page u = t / T at physical page
 * page_table[u], slot t % T.  Grouping never changes A_i (Figure 2: all
 * selected edges are retained), so this definition is the result of the union
 * kernel for any grouping.
 *
 * The grouping reference implements the bounded page-affinity rule read from
 * the Abstract (a search of bounded cost on the GPU turns the affinity of the
 * queries' selected pages into lists of query IDs) and Figure 2 (logical page
 * visits and masked query-page slots), with sets held as sorted integer arrays:
 *   per KV head h and query i, S(i) = sorted distinct valid pages of the g
 *   rows topk[h*g + j][i][:];  fixed windows [w*W, (w+1)*W) of query IDs;
 *   inside a window: seed = smallest unassigned ID, U = S(seed); while the
 *   group has fewer than max_group members and unassigned queries remain,
 *   add the candidate c with the fewest pages outside U (ties: smallest ID)
 *   and set U = U + S(c).  Members are listed ascending, groups by window then
 *   seed, unions ascending.  Row bit r = rank(member)*g + j of a union page is
 *   set iff the page is in row topk[h*g+j][member].
 *   Counters per KV head: visits = sum |U|; masked_row_slots = sum over groups
 *   and rows of (|U| - |S_j(m)|); masked_query_slots = sum over groups and
 *   members of (|U| - |S(m)|); page_edges = sum_i |S(i)|.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2 };
enum { ORC_OK = 0, ORC_EARG = 1, ORC_EPAGE = 2, ORC_ECAP = 3, ORC_EMEM = 4 };

/* ---------------------------------------------------------------- decoders */

/* bfloat16: the upper 16 bits of an IEEE binary32; widening is exact. */
static double orc_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* OCP FP8 E4M3 by its definition: 1 sign bit, 4 exponent bits (bias 7),
 * 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); the pattern
 * S.1111.111 is NaN; there are no infinities (largest finite 448). */
double oracle_e4m3_decode(uint8_t b) {
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

double oracle_bf16_decode(uint16_t b) { return orc_bf16(b); }

static double load_elem(const void* base, int dtype, size_t idx, double scale) {
    switch (dtype) {
    case ORC_F32: return (double)((const float*)base)[idx];
    case ORC_BF16: return orc_bf16(((const uint16_t*)base)[idx]);
    default: return oracle_e4m3_decode(((const uint8_t*)base)[idx]) * scale;
    }
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* sorted distinct valid entries of one TopK row; returns count or -1 on a bad id */
static int row_set(const int32_t* row, int K, int P, int32_t* out) {
    int n = 0;
    for (int k = 0; k < K; ++k) {
        int32_t p = row[k];
        if (p == -1) continue;
        if (p < 0 || p >= P) return -1;
        out[n++] = p;
    }
    qsort(out, (size_t)n, sizeof(int32_t), cmp_i32);
    int m = 0;
    for (int k = 0; k < n; ++k)
        if (m == 0 || out[m - 1] != out[k]) out[m++] = out[k];
    return m;
}

/* ------------------------------------------------------------- attention */

/*
 * Sparse attention for a list of (Q head, query) rows.
 * rows: nrows entries r = h' * Nq + i (NULL = every row, in [i][h'] order of O).
 * O: [nrows][d] (or [Nq][Hq][d] when rows == NULL), lse: same indexing, natural log.
 * Empty support gives O = 0 and lse = -inf.
 */
int oracle_sparse_attn(const void* Q, int q_dtype, const void* Kc, const void* Vc, int kv_dtype,
                       const float* k_scale, const float* v_scale,
                       const int32_t* page_table, int num_logical_pages, int P_phys, int T,
                       const int32_t* topk, int K, const int32_t* q_pos, int kv_len,
                       int Hq, int Hkv, int Nq, int d, double softmax_scale,
                       const int64_t* rows, int64_t nrows, double* O, double* lse, int nthreads) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq < 0 || d <= 0 || T <= 0 || K < 0) return ORC_EARG;
    if (kv_dtype == ORC_E4M3 && (!k_scale || !v_scale)) return ORC_EARG;
    const int g = Hq / Hkv;
    const int64_t total = rows ? nrows : (int64_t)Hq * Nq;
    int err = ORC_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        int32_t* pages = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
        size_t cap = (size_t)(K > 0 ? K : 1) * (size_t)T;
        double* s = (double*)malloc(sizeof(double) * cap);
        int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * cap);
        double* q = (double*)malloc(sizeof(double) * (size_t)d);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
        for (int64_t n = 0; n < total; ++n) {
            int64_t r = rows ? rows[n] : ((n % Hq) * (int64_t)Nq + n / Hq);
            int hq = (int)(r / Nq), i = (int)(r % Nq);
            int h = hq / g;
            double* out = O + (size_t)n * d;
            double* out_lse = lse ? lse + n : NULL;
            if (!rows) {  /* O laid out [Nq][Hq][d] */
                out = O + ((size_t)i * Hq + hq) * d;
                out_lse = lse ? lse + (size_t)i * Hq + hq : NULL;
            }
            int np = row_set(topk + ((size_t)hq * Nq + i) * K, K, num_logical_pages, pages);
            if (np < 0) {
#pragma omp atomic write
                err = ORC_EPAGE;
                continue;
            }
            for (int c = 0; c < d; ++c)
                q[c] = load_elem(Q, q_dtype, ((size_t)i * Hq + hq) * d + c, 1.0);
            double ks = (kv_dtype == ORC_E4M3) ? (double)k_scale[h] : 1.0;
            double vs = (kv_dtype == ORC_E4M3) ? (double)v_scale[h] : 1.0;
            /* pass 1: scores of the visible tokens and their maximum */
            int64_t nt = 0;
            double mx = -INFINITY;
            for (int a = 0; a < np; ++a) {
                int u = pages[a];
                int phys = page_table[u];
                if (phys < 0 || phys >= P_phys) {
#pragma omp atomic write
                    err = ORC_EPAGE;
                    continue;
                }
                for (int o = 0; o < T; ++o) {
                    int64_t t = (int64_t)u * T + o;
                    if (t >= kv_len || t > q_pos[i]) continue;
                    size_t kb = (((size_t)phys * Hkv + h) * T + o) * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += q[c] * load_elem(Kc, kv_dtype, kb + c, ks);
                    s[nt] = dot * softmax_scale;
                    tok[nt] = ((int64_t)phys * Hkv + h) * T + o;
                    if (s[nt] > mx) mx = s[nt];
                    ++nt;
                }
            }
            /* pass 2: exponential sum and weighted sum of V */
            for (int c = 0; c < d; ++c) acc[c] = 0.0;
            double l = 0.0;
            for (int64_t a = 0; a < nt; ++a) {
                double w = exp(s[a] - mx);
                l += w;
                size_t vb = (size_t)tok[a] * d;
                for (int c = 0; c < d; ++c) acc[c] += w * load_elem(Vc, kv_dtype, vb + c, vs);
            }
            for (int c = 0; c < d; ++c) out[c] = (nt > 0) ? acc[c] / l : 0.0;
            if (out_lse) *out_lse = (nt > 0) ? mx + log(l) : -INFINITY;
        }
        free(pages); free(s); free(tok); free(q); free(acc);
    }
    return err;
}

/* ------------------------------------------------------- grouping reference */

typedef struct { int32_t* v; int n; } iset;

/* |a \ b| for sorted distinct arrays */
static int set_minus_count(const iset* a, const iset* b) {
    int i = 0, j = 0, c = 0;
    while (i < a->n) {
        if (j >= b->n || a->v[i] < b->v[j]) { ++c; ++i; }
        else if (a->v[i] == b->v[j]) { ++i; ++j; }
        else ++j;
    }
    return c;
}

/* u = u + a (sorted union), tmp must hold u->n + a->n */
static void set_union_into(iset* u, const iset* a, int32_t* tmp) {
    int i = 0, j = 0, n = 0;
    while (i < u->n || j < a->n) {
        if (j >= a->n || (i < u->n && u->v[i] < a->v[j])) tmp[n++] = u->v[i++];
        else if (i >= u->n || a->v[j] < u->v[i]) tmp[n++] = a->v[j++];
        else { tmp[n++] = u->v[i++]; ++j; }
    }
    memcpy(u->v, tmp, sizeof(int32_t) * (size_t)n);
    u->n = n;
}

static int set_has(const iset* a, int32_t p) {
    int lo = 0, hi = a->n - 1;
    while (lo <= hi) {
        int mid = (lo + hi) / 2;
        if (a->v[mid] == p) return 1;
        if (a->v[mid] < p) lo = mid + 1; else hi = mid - 1;
    }
    return 0;
}

/*
 * Union page lists, row masks and counters for a given partition of the
 * queries of every KV head into groups (n_groups, group_ptr, members as
 * produced by the grouping rule, or any other partition with at most 64 rows
 * per group).  union_ptr[h][k] are absolute offsets into union_pages/row_mask;
 * the regions of the KV heads follow each other in head order.
 */
int oracle_build_unions(const int32_t* topk, int Hq, int Hkv, int Nq, int K, int P,
                        const int32_t* n_groups, const int32_t* group_ptr, const int32_t* members,
                        int32_t* union_ptr, int32_t* union_pages, uint64_t* row_mask,
                        int64_t cap, int64_t* counters) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq < 0 || K < 0 || P <= 0) return ORC_EARG;
    const int g = Hq / Hkv;
    int64_t off = 0;
    int32_t* U = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (size_t)P * 2 + 8);
    int32_t* buf = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K * g + 1) * 65);
    if (!U || !tmp || !buf) { free(U); free(tmp); free(buf); return ORC_EMEM; }
    int rc = ORC_OK;
    for (int h = 0; h < Hkv && rc == ORC_OK; ++h) {
        int64_t* ctr = counters + 4 * h;
        ctr[0] = ctr[1] = ctr[2] = ctr[3] = 0;
        const int32_t* gp = group_ptr + (size_t)h * (Nq + 1);
        const int32_t* mem = members + (size_t)h * Nq;
        int32_t* up = union_ptr + (size_t)h * (Nq + 1);
        for (int q = 0; q < Nq && rc == ORC_OK; ++q) {  /* page edges: sum |S(i)| */
            iset s = { buf, 0 };
            for (int j = 0; j < g; ++j) {
                int n = row_set(topk + ((size_t)(h * g + j) * Nq + q) * K, K, P, buf + s.n);
                if (n < 0) { rc = ORC_EPAGE; break; }
                s.n += n;
            }
            if (rc) break;
            qsort(buf, (size_t)s.n, sizeof(int32_t), cmp_i32);
            int m = 0;
            for (int k = 0; k < s.n; ++k) if (m == 0 || buf[m - 1] != buf[k]) buf[m++] = buf[k];
            ctr[3] += m;
        }
        for (int G = 0; G < n_groups[h] && rc == ORC_OK; ++G) {
            int nm = gp[G + 1] - gp[G];
            if (nm * g > 64) { rc = ORC_EARG; break; }
            iset u = { U, 0 };
            /* rows of the group: row r = rank*g + j -> its own set */
            iset rs[64];
            int used = 0;
            for (int m = 0; m < nm && rc == ORC_OK; ++m) {
                int qi = mem[gp[G] + m];
                for (int j = 0; j < g; ++j) {
                    int32_t* dst = buf + (size_t)used;
                    int n = row_set(topk + ((size_t)(h * g + j) * Nq + qi) * K, K, P, dst);
                    if (n < 0) { rc = ORC_EPAGE; break; }
                    rs[m * g + j].v = dst;
                    rs[m * g + j].n = n;
                    used += n;
                    set_union_into(&u, &rs[m * g + j], tmp);
                }
            }
            if (rc) break;
            up[G] = (int32_t)off;
            if (off + u.n > cap) { rc = ORC_ECAP; break; }
            for (int a = 0; a < u.n; ++a) {
                uint64_t mk = 0;
                for (int r = 0; r < nm * g; ++r)
                    if (set_has(&rs[r], u.v[a])) mk |= (uint64_t)1 << r;
                union_pages[off + a] = u.v[a];
                row_mask[off + a] = mk;
            }
            ctr[0] += u.n;
            for (int m = 0; m < nm; ++m) {
                /* |S(m)| = union pages present in any of the member's g rows */
                int cnt = 0;
                for (int a = 0; a < u.n; ++a) {
                    int any = 0;
                    for (int j = 0; j < g; ++j) any |= set_has(&rs[m * g + j], u.v[a]);
                    cnt += any;
                }
                ctr[2] += u.n - cnt;
                for (int j = 0; j < g; ++j) ctr[1] += u.n - rs[m * g + j].n;
            }
            off += u.n;
        }
        if (rc == ORC_OK) up[n_groups[h]] = (int32_t)off;
    }
    free(U); free(tmp); free(buf);
    return rc;
}

/* Greedy windowed page-affinity grouping followed by the union build. */
int oracle_group(const int32_t* topk, int Hq, int Hkv, int Nq, int K, int P,
                 int max_group, int window,
                 int32_t* n_groups, int32_t* group_ptr, int32_t* members,
                 int32_t* union_ptr, int32_t* union_pages, uint64_t* row_mask,
                 int64_t cap, int64_t* counters) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq < 0 || K < 0 || P <= 0) return ORC_EARG;
    if (max_group < 1 || window < max_group || window % max_group) return ORC_EARG;
    const int g = Hq / Hkv;
    int32_t* store = (int32_t*)malloc(sizeof(int32_t) * ((size_t)window * K * g + 1));
    iset* S = (iset*)malloc(sizeof(iset) * (size_t)window);
    int32_t* U = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
    int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (size_t)P * 2 + 8);
    char* taken = (char*)malloc((size_t)window);
    int32_t grp[64];
    if (!store || !S || !U || !tmp || !taken) {
        free(store); free(S); free(U); free(tmp); free(taken);
        return ORC_EMEM;
    }
    int rc = ORC_OK;
    for (int h = 0; h < Hkv && rc == ORC_OK; ++h) {
        int32_t* gp = group_ptr + (size_t)h * (Nq + 1);
        int32_t* mem = members + (size_t)h * Nq;
        int ng = 0, nmem = 0;
        gp[0] = 0;
        for (int w0 = 0; w0 < Nq && rc == ORC_OK; w0 += window) {
            int nw = (Nq - w0 < window) ? Nq - w0 : window;
            size_t used = 0;
            for (int a = 0; a < nw; ++a) {  /* canonical sets S(i) */
                S[a].v = store + used;
                int n = 0;
                for (int j = 0; j < g; ++j) {
                    int c = row_set(topk + ((size_t)(h * g + j) * Nq + w0 + a) * K, K, P,
                                    S[a].v + n);
                    if (c < 0) { rc = ORC_EPAGE; break; }
                    n += c;
                }
                if (rc) break;
                qsort(S[a].v, (size_t)n, sizeof(int32_t), cmp_i32);
                int m = 0;
                for (int k = 0; k < n; ++k) if (m == 0 || S[a].v[m - 1] != S[a].v[k]) S[a].v[m++] = S[a].v[k];
                S[a].n = m;
                used += (size_t)m;
                taken[a] = 0;
            }
            if (rc) break;
            for (int seed = 0; seed < nw; ++seed) {
                if (taken[seed]) continue;
                iset u = { U, S[seed].n };
                memcpy(U, S[seed].v, sizeof(int32_t) * (size_t)S[seed].n);
                taken[seed] = 1;
                int cnt = 1;
                grp[0] = seed;
                while (cnt < max_group) {
                    int best = -1, bestc = 0;
                    for (int c = seed + 1; c < nw; ++c) {
                        if (taken[c]) continue;
                        int nc = set_minus_count(&S[c], &u);
                        if (best < 0 || nc < bestc) { best = c; bestc = nc; }
                    }
                    if (best < 0) break;
                    taken[best] = 1;
                    set_union_into(&u, &S[best], tmp);
                    grp[cnt++] = best;
                }
                qsort(grp, (size_t)cnt, sizeof(int32_t), cmp_i32);
                for (int m = 0; m < cnt; ++m) mem[nmem++] = w0 + grp[m];
                gp[++ng] = nmem;
            }
        }
        n_groups[h] = ng;
    }
    free(store); free(S); free(U); free(tmp); free(taken);
    if (rc) return rc;
    return oracle_build_unions(topk, Hq, Hkv, Nq, K, P, n_groups, group_ptr, members,
                               union_ptr, union_pages, row_mask, cap, counters);
}

/*
 * Bundles (an execution-level packing with no counterpart on the pages): per
 * KV head, the groups in order are cut into windows of wb groups; inside a
 * window a bundle is seeded with the first unbundled group and grown, up to
 * `slots` groups, by the group with the smallest  new - 2 * shared , new
 * being the pages its union adds to the bundle union and shared the pages
 * of its union already in it (ties: smallest index).  Groups of a bundle are listed
 * ascending (slot order).  Row of slot j, member rank m, head offset jj:
 * j*rs + m*g + jj.  The 128-bit mask of a bundle page has the group's row
 * mask of that page at bit offset j*rs.
 *   rs = smallest power of two >= max_group*g; slots = 128/rs;
 *   wb = max(slots, (bundle_window/slots)*slots).
 * Inputs are the group arrays (as produced by oracle_group or
 * oracle_build_unions).  bmask holds 4 uint32 per entry; bqid has 128/g
 * entries per bundle slot of [Hkv][Nq].
 */
int oracle_bundle(int Hq, int Hkv, int Nq, int max_group, int bundle_window,
                  const int32_t* n_groups, const int32_t* group_ptr, const int32_t* members,
                  const int32_t* union_ptr, const int32_t* union_pages, const uint64_t* row_mask,
                  int32_t* n_bundles, int32_t* bundle_ptr, int32_t* bundle_groups,
                  int32_t* bunion_ptr, int32_t* bunion_pages, uint32_t* bmask, int32_t* bqid,
                  int64_t cap, int64_t* bcounters) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq < 0 || max_group < 1) return ORC_EARG;
    const int g = Hq / Hkv;
    int rs = 1;
    while (rs < max_group * g) rs <<= 1;
    if (rs > 32) return ORC_EARG;
    const int slots = 128 / rs;
    int wb = bundle_window > 0 ? bundle_window : 64;
    wb = (wb / slots) * slots;
    if (wb < slots) wb = slots;
    const int mq = 128 / g;
    int64_t off = 0;
    int rc = ORC_OK;
    int pmax = 1;
    for (int64_t e = 0; e < (Hkv > 0 ? union_ptr[(size_t)(Hkv - 1) * (Nq + 1) + n_groups[Hkv - 1]] : 0); ++e)
        if (union_pages[e] + 1 > pmax) pmax = union_pages[e] + 1;
    int32_t* U = (int32_t*)malloc(sizeof(int32_t) * (size_t)pmax);
    int32_t* tmp = (int32_t*)malloc(sizeof(int32_t) * (size_t)pmax * 2 + 8);
    char* taken = (char*)malloc((size_t)(wb > 0 ? wb : 1));
    int32_t grp[128];
    if (!U || !tmp || !taken) { free(U); free(tmp); free(taken); return ORC_EMEM; }
    for (int h = 0; h < Hkv && rc == ORC_OK; ++h) {
        const int32_t* gp = group_ptr + (size_t)h * (Nq + 1);
        const int32_t* up = union_ptr + (size_t)h * (Nq + 1);
        int32_t* bp = bundle_ptr + (size_t)h * (Nq + 1);
        int32_t* bu = bunion_ptr + (size_t)h * (Nq + 1);
        int nb = 0, nbg = 0;
        int64_t visits = 0;
        bp[0] = 0;
        const int ng = n_groups[h];
        for (int w0 = 0; w0 < ng && rc == ORC_OK; w0 += wb) {
            const int nw = (ng - w0 < wb) ? ng - w0 : wb;
            for (int a = 0; a < nw; ++a) taken[a] = 0;
            for (int seed = 0; seed < nw; ++seed) {
                if (taken[seed]) continue;
                iset u = { U, up[w0 + seed + 1] - up[w0 + seed] };
                memcpy(U, union_pages + up[w0 + seed], sizeof(int32_t) * (size_t)u.n);
                taken[seed] = 1;
                int cnt = 1;
                grp[0] = seed;
                while (cnt < slots) {
                    int best = -1, bestc = 0;
                    for (int c = seed + 1; c < nw; ++c) {
                        if (taken[c]) continue;
                        iset sc = { (int32_t*)union_pages + up[w0 + c], up[w0 + c + 1] - up[w0 + c] };
                        /* new pages counted against pages already shared with the bundle union:
                         * new - 2 * shared = 3 * new - 2 * |S(c)| */
                        int nc = 3 * set_minus_count(&sc, &u) - 2 * sc.n;
                        if (best < 0 || nc < bestc) { best = c; bestc = nc; }
                    }
                    if (best < 0) break;
                    taken[best] = 1;
                    iset sb = { (int32_t*)union_pages + up[w0 + best], up[w0 + best + 1] - up[w0 + best] };
                    set_union_into(&u, &sb, tmp);
                    grp[cnt++] = best;
                }
                qsort(grp, (size_t)cnt, sizeof(int32_t), cmp_i32);
                /* emit */
                bu[nb] = (int32_t)off;
                if (off + u.n > cap) { rc = ORC_ECAP; break; }
                int32_t* q = bqid + ((size_t)h * Nq + nb) * mq;
                for (int k = 0; k < mq; ++k) q[k] = -1;
                for (int j = 0; j < cnt; ++j) {
                    const int gi = w0 + grp[j];
                    bundle_groups[(size_t)h * Nq + nbg + j] = gi;
                    for (int m = 0; m < gp[gi + 1] - gp[gi]; ++m)
                        q[j * (rs / g) + m] = members[(size_t)h * Nq + gp[gi] + m];
                }
                for (int a = 0; a < u.n; ++a) {
                    uint32_t mk[4] = {0, 0, 0, 0};
                    for (int j = 0; j < cnt; ++j) {
                        const int gi = w0 + grp[j];
                        /* the group's entry for this page, if any */
                        int lo = up[gi], hi = up[gi + 1] - 1, at = -1;
                        while (lo <= hi) {
                            int mid = (lo + hi) / 2;
                            if (union_pages[mid] == u.v[a]) { at = mid; break; }
                            if (union_pages[mid] < u.v[a]) lo = mid + 1; else hi = mid - 1;
                        }
                        if (at < 0) continue;
                        const uint64_t rm = row_mask[at];
                        for (int r = 0; r < rs; ++r)
                            if ((rm >> r) & 1) {
                                const int row = j * rs + r;
                                mk[row >> 5] |= 1u << (row & 31);
                            }
                    }
                    bunion_pages[off + a] = u.v[a];
                    for (int k = 0; k < 4; ++k) bmask[(off + a) * 4 + k] = mk[k];
                }
                off += u.n;
                visits += u.n;
                nbg += cnt;
                bp[++nb] = nbg;
            }
        }
        if (rc) break;
        bu[nb] = (int32_t)off;
        n_bundles[h] = nb;
        bcounters[2 * h] = visits;
        bcounters[2 * h + 1] = nb;
    }
    free(U); free(tmp); free(taken);
    return rc;
}
