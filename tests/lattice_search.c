/*
 * lattice_search.c -- exhaustive nearest-point search for the E8, D4 and A2 lattices, used by the
 * tests to pin the oracle's closest-point rules on millions of inputs.  Test infrastructure only;
 * it shares nothing with the oracle or the CUDA library.
 *
 * Method: every lattice point within the covering radius of the input is a candidate (the nearest
 * point always is one), enumerated coordinate by coordinate by depth-first search in binary64;
 * a branch is abandoned once its partial squared distance exceeds the best complete distance
 * found so far plus `tol`.  All points whose distance is within `tol` of the minimum are kept, so
 * the caller learns whether the nearest point is unique and which points tie with it.
 *
 * Lattices, as the codec's integer embeddings:
 *   E8 in doubled coordinates z = 2u: integer vectors with all coordinates of one parity and a
 *      sum divisible by 4; covering radius 2 (1 in u units), so |z_i - p_i| <= 2.
 *   D4 in u units: integer vectors with an even sum; covering radius 1.
 *   A2 in u units with minimum distance 1: (a + b/2, b sqrt(3)/2), a, b integers; covering
 *      radius 1/sqrt(3).  The embedding returned is (P, Q) = (2a + b, b).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define MAXKEEP 512

typedef struct {
    double best;          /* smallest complete squared distance seen */
    double tol;
    int nkeep;
    double kd[MAXKEEP];   /* kept candidates: squared distance and point */
    int32_t kp[MAXKEEP][8];
} search_t;

static void keep(search_t* s, const int32_t* p, int d, double dist)
{
    if (dist < s->best) s->best = dist;
    if (s->nkeep < MAXKEEP) {
        s->kd[s->nkeep] = dist;
        memcpy(s->kp[s->nkeep], p, sizeof(int32_t) * d);
        s->nkeep++;
    }
}

static void dfs_e8(const double* z, int i, int par, int32_t* p, double part, int64_t sum, search_t* s)
{
    if (i == 8) {
        if (((sum % 4) + 4) % 4 == 0) keep(s, p, 8, part);
        return;
    }
    int lo = (int)ceil(z[i] - 2.0), hi = (int)floor(z[i] + 2.0);
    for (int v = lo; v <= hi; ++v) {
        if ((((v % 2) + 2) % 2) != par) continue;
        double t = z[i] - (double)v;
        double np = part + t * t;
        if (np > s->best + s->tol) continue;
        p[i] = v;
        dfs_e8(z, i + 1, par, p, np, sum + v, s);
    }
}

static void dfs_d4(const double* u, int i, int32_t* p, double part, int64_t sum, search_t* s)
{
    if (i == 4) {
        if (((sum % 2) + 2) % 2 == 0) keep(s, p, 4, part);
        return;
    }
    int lo = (int)ceil(u[i] - 1.0), hi = (int)floor(u[i] + 1.0);
    for (int v = lo; v <= hi; ++v) {
        double t = u[i] - (double)v;
        double np = part + t * t;
        if (np > s->best + s->tol) continue;
        p[i] = v;
        dfs_d4(u, i + 1, p, np, sum + v, s);
    }
}

/* finish: keep only the candidates within tol of the final minimum */
static int finish(search_t* s, int d, double* best_d, int32_t* best_p, int32_t* ties)
{
    int n = 0, first = -1;
    for (int k = 0; k < s->nkeep; ++k)
        if (s->kd[k] <= s->best + s->tol) {
            if (first < 0 || s->kd[k] < s->kd[first]) first = k;
            n++;
        }
    *best_d = s->kd[first];
    memcpy(best_p, s->kp[first], sizeof(int32_t) * d);
    (void)ties;
    return n;
}

/*
 * For each of m inputs (binary32, u units, d coordinates each): the minimum squared distance
 * (u units, binary64) in best_d[m], a nearest point (integer embedding) in best_p[m * d], and in
 * count[m] the number of lattice points within tol (u^2 units) of the minimum.  Returns 0, or -1
 * for an unknown lattice.  lattice: 1 A2, 2 D4, 3 E8 (the codec's numbering).
 */
int ls_nearest(int lattice, const float* u, int64_t m, double tol, double* best_d, int32_t* best_p, int32_t* count)
{
    for (int64_t b = 0; b < m; ++b) {
        search_t s;
        s.nkeep = 0;
        int32_t p[8];
        if (lattice == 3) {
            double z[8];
            for (int i = 0; i < 8; ++i) z[i] = 2.0 * (double)u[8 * b + i];
            s.tol = 4.0 * tol;
            s.best = 4.0 + 1e-9;   /* covering radius^2 in doubled units */
            dfs_e8(z, 0, 0, p, 0.0, 0, &s);
            dfs_e8(z, 0, 1, p, 0.0, 0, &s);
            double bd;
            count[b] = finish(&s, 8, &bd, best_p + 8 * b, 0);
            best_d[b] = bd / 4.0;
        } else if (lattice == 2) {
            double x[4];
            for (int i = 0; i < 4; ++i) x[i] = (double)u[4 * b + i];
            s.tol = tol;
            s.best = 1.0 + 1e-9;
            dfs_d4(x, 0, p, 0.0, 0, &s);
            double bd;
            count[b] = finish(&s, 4, &bd, best_p + 4 * b, 0);
            best_d[b] = bd;
        } else if (lattice == 1) {
            const double h = sqrt(3.0) / 2.0, R = 1.0 / sqrt(3.0) + 1e-9;
            double x = (double)u[2 * b], y = (double)u[2 * b + 1];
            s.tol = tol;
            s.best = R * R;
            int blo = (int)ceil((y - R) / h), bhi = (int)floor((y + R) / h);
            for (int bb = blo; bb <= bhi; ++bb) {
                double ty = y - bb * h;
                int alo = (int)ceil(x - bb / 2.0 - R), ahi = (int)floor(x - bb / 2.0 + R);
                for (int aa = alo; aa <= ahi; ++aa) {
                    double tx = x - (aa + bb / 2.0);
                    double dd = tx * tx + ty * ty;
                    if (dd > s.best + s.tol) continue;
                    p[0] = 2 * aa + bb;
                    p[1] = bb;
                    keep(&s, p, 2, dd);
                }
            }
            double bd;
            count[b] = finish(&s, 2, &bd, best_p + 2 * b, 0);
            best_d[b] = bd;
        } else {
            return -1;
        }
    }
    return 0;
}
