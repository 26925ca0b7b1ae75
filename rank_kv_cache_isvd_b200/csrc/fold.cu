// Block-incremental truncated-SVD update ("fold") of one (layer, sequence, kv-head, path) unit.
//
// iS-KV summary, "Block-Incremental Decoding Updates", steps 1-3, for history A = U Sigma B^T
// (k components, coordinates C = U Sigma stored) and pending block F (b rows of the window):
//   1. S = F B, E = F - S B^T; orthonormal residual basis P (d x p) from a Householder QR of
//      [B, E^T] (its columns after the first k), p = min(b, d - k). The QR runs over B's columns
//      first, which re-orthogonalises E against B to rounding (the oracle's second projection pass).
//   2. Z = [[Sigma, 0], [S, F P]], (k + b) x (k + p); with P from that QR, F P = E P is the
//      transpose of the QR's trailing R block for the rows that entered it.
//   3. (G, Sigma+, H) = SVD_r(Z): Z is first reduced to its triangular factor R (Householder,
//      Q discarded; R^T R = Z^T Z), then one-sided (Hestenes) Jacobi runs on the columns of R^T:
//      at convergence the columns of R^T J are orthogonal, their norms are the singular values
//      and the normalised columns are the right singular vectors H of Z, so J is never accumulated;
//      B+ = [B P] H, the old coordinates move by H[:k] (rotate_kernel) and the new rows'
//      coordinates are F B+ (bottom block of U+ Sigma+, since Z H = G Sigma+).
// One CTA (256 threads) per unit and path (blockIdx.y = path), everything on chip (b <= 128).
#include "iskv_internal.cuh"

namespace iskv {

constexpr int FT = 256;                       // threads
constexpr int FW = FT / 32;                   // warps
constexpr int JL = 16;                        // lanes per Jacobi column group
constexpr int SS = 132;                       // column stride of the Jacobi staging area
constexpr float JACOBI_TOL = 4e-6f;           // rotate while |a.b| > tol |a| |b|
constexpr float JACOBI_ZERO = 1e-10f;         // columns with |a|^2 <= this * ||Z||_F^2 are noise

// shared memory (floats)
constexpr int OFF_A = 0;                                  // F/E rows -> [P | B_old] -> F rows
constexpr int OFF_B = OFF_A + 128 * LDS;                  // Y = [S | T] rows
constexpr int STAGE_FLOATS = 2 * 128 * SS;                // two Jacobi staging buffers of 128
                                                          // columns (overlay B and C)
constexpr int C_FLOATS = STAGE_FLOATS - 128 * LDS;        // QR columns -> Sigma columns
constexpr int OFF_C = OFF_B + 128 * LDS;
constexpr int OFF_TAU = OFF_C + C_FLOATS;
constexpr int OFF_SIG = OFF_TAU + 128;
constexpr int OFF_NRM = OFF_SIG + 128;                    // [256] column norms
constexpr int OFF_SNRM = OFF_NRM + 256;                   // [2][128] staged squared norms
constexpr int OFF_SCR = OFF_SNRM + 256;                   // per-warp scratch, 128 floats each
constexpr int OFF_INT = OFF_SCR + FW * 128;               // ints: sel[256], flags[4]
constexpr int SMEM_FLOATS = OFF_INT + 256 + 4;
static_assert(C_FLOATS >= 128 * LDS, "QR matrix must fit");

size_t fold_smem_bytes() { return (size_t)SMEM_FLOATS * sizeof(float); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float group_sum(float v) {   // over the 16 lanes of a Jacobi group
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    return v;
}

// Rotation parameters of one Hestenes step for columns with squared norms nx, ny and inner
// product g: t = tan(theta) of the rotation [[c, s], [-s, c]] that makes the pair orthogonal, or
// t = 0 (identity) when |g| <= tol |x| |y|. Returns (s, dc) with dc = 1 - c formed directly: for
// |t| < sqrt(eps) c rounds to 1 while s = t, and a rounded rotation would inflate the norms by
// t^2/2 every time (a systematic bias over thousands of rotations). With dc and s derived from
// the same 1/sqrt(1 + t^2), c^2 + s^2 - 1 = O(eps t^2), so approximate reciprocals and square
// roots keep tiny rotations norm-preserving. Pairs with a column whose squared norm is at most
// `floor2` are left alone: such columns hold rounding noise only (when the core has more rows
// than columns, Z^T has more columns than dimensions and the surplus converges to zero), and
// their normalised inner products would otherwise stay O(1) for ever.
__device__ __forceinline__ void jparams(float g, float nx, float ny, float floor2, float &t,
                                        float &s, float &dc) {
    const bool doit = g * g > (JACOBI_TOL * JACOBI_TOL) * nx * ny && fminf(nx, ny) > floor2;
    const float gg = doit ? g : 1.f;
    const float zeta = __fdividef(ny - nx, 2.f * gg);
    const float az = fminf(fabsf(zeta), 1e18f);
    const float q = fmaf(az, az, 1.f);
    const float t0 = __fdividef(1.f, az + q * rsqrtf(q));
    t = doit ? copysignf(t0, zeta) : 0.f;
    const float ri = rsqrtf(fmaf(t, t, 1.f));           // c = 1 / sqrt(1 + t^2)
    s = t * ri;
    dc = __fdividef(t * t * ri * ri, 1.f + ri);          // 1 - c
}

// Dot product of a lane's RPL rows of two columns, two rows per packed fp32x2 FMA.
template <int RPL>
__device__ __forceinline__ float jdot(const float (&x)[RPL], const float (&y)[RPL]) {
    float2 g2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i + 1 < RPL; i += 2)
        g2 = __ffma2_rn(make_float2(x[i], x[i + 1]), make_float2(y[i], y[i + 1]), g2);
    if (RPL & 1) g2.x = fmaf(x[RPL - 1], y[RPL - 1], g2.x);
    return g2.x + g2.y;
}

// x <- x - dc x - sn y, y <- y - dc y + sn x over a lane's RPL rows (packed fp32x2 FMAs).
template <int RPL>
__device__ __forceinline__ void jturn(float (&x)[RPL], float (&y)[RPL], float sn, float dc) {
    const float2 ndc = make_float2(-dc, -dc), nsn = make_float2(-sn, -sn), psn = make_float2(sn, sn);
#pragma unroll
    for (int i = 0; i + 1 < RPL; i += 2) {
        const float2 xi = make_float2(x[i], x[i + 1]), yi = make_float2(y[i], y[i + 1]);
        const float2 xo = __ffma2_rn(nsn, yi, __ffma2_rn(ndc, xi, xi));
        const float2 yo = __ffma2_rn(psn, xi, __ffma2_rn(ndc, yi, yi));
        x[i] = xo.x;
        x[i + 1] = xo.y;
        y[i] = yo.x;
        y[i + 1] = yo.y;
    }
    if (RPL & 1) {
        const float xi = x[RPL - 1], yi = y[RPL - 1];
        x[RPL - 1] = fmaf(-sn, yi, fmaf(-dc, xi, xi));
        y[RPL - 1] = fmaf(sn, xi, fmaf(-dc, yi, yi));
    }
}

// Rotates HC disjoint column pairs (x_j, y_(j+S) mod HC) of a lane group at once: the dot
// products, their reductions and the rotation parameters of all pairs overlap (no branches).
template <int HC, int RPL, int S>
__device__ __forceinline__ void jcross(float (&xa)[HC][RPL], float (&xb)[HC][RPL], float (&na)[HC],
                                       float (&nb)[HC], float floor2, int &rotated) {
    float g[HC];
#pragma unroll
    for (int j = 0; j < HC; ++j) g[j] = jdot<RPL>(xa[j], xb[(j + S) % HC]);
#pragma unroll
    for (int o = 1; o < JL; o <<= 1)
#pragma unroll
        for (int j = 0; j < HC; ++j) g[j] += __shfl_xor_sync(0xffffffffu, g[j], o);
#pragma unroll
    for (int j = 0; j < HC; ++j) {
        const int jb = (j + S) % HC;
        float t, sn, dc;
        jparams(g[j], na[j], nb[jb], floor2, t, sn, dc);
        jturn<RPL>(xa[j], xb[jb], sn, dc);
        na[j] = fmaxf(na[j] - t * g[j], 0.f);
        nb[jb] = fmaxf(nb[jb] + t * g[j], 0.f);
        rotated |= (t != 0.f);
    }
}

// One rotation of the pair (x, y) within a slot (used in round 0 of a sweep).
template <int RPL>
__device__ __forceinline__ void jrot(float (&x)[RPL], float (&y)[RPL], float &nx, float &ny,
                                     float floor2, int &rotated) {
    const float g = group_sum(jdot<RPL>(x, y));
    float t, sn, dc;
    jparams(g, nx, ny, floor2, t, sn, dc);
    jturn<RPL>(x, y, sn, dc);
    nx = fmaxf(nx - t * g, 0.f);
    ny = fmaxf(ny + t * g, 0.f);
    rotated |= (t != 0.f);
}

template <int HC, int RPL, int S>
struct JCrossAll {
    __device__ __forceinline__ static void run(float (&xa)[HC][RPL], float (&xb)[HC][RPL],
                                               float (&na)[HC], float (&nb)[HC], float floor2,
                                               int &rotated) {
        jcross<HC, RPL, S>(xa, xb, na, nb, floor2, rotated);
        JCrossAll<HC, RPL, S + 1>::run(xa, xb, na, nb, floor2, rotated);
    }
};
template <int HC, int RPL>
struct JCrossAll<HC, RPL, HC> {
    __device__ __forceinline__ static void run(float (&)[HC][RPL], float (&)[HC][RPL],
                                               float (&)[HC], float (&)[HC], float, int &) {}
};

// Register-resident one-sided Jacobi on N <= 2 ng HC columns of length n <= 16 RPL, where
// ng = ceil(N / (2 HC)) <= 16 column groups are active. Group g (16 lanes) holds slots top[g] and
// bottom[g] of HC columns each; lane l holds rows [RPL l, RPL l + RPL). Each sweep is the
// round-robin (circle) tournament on the 2 ng slots: 2 ng - 1 rounds, every slot pair meets once;
// columns within a slot are rotated in round 0. Between rounds the slots move through the
// staging area: top[0] stays, top[i] -> top[i+1], top[ng-1] -> bottom[ng-1],
// bottom[i] -> bottom[i-1], bottom[0] -> top[1].
// On return the final columns are in `stage` (column (pos*HC + j), stride SS, 2 ng HC columns)
// with their norms in nrm_out; returns the number of sweeps (negative if the cap was reached).
template <int HC, int RPL>
__device__ __noinline__ int jacobi_regs(const float *sB, const float *sC, int k, int N, int n,
                                        float *stage, float *stage_n, float *nrm_out) {
    const int tid = threadIdx.x;
    const int grp = tid / JL, gl = tid % JL;
    const int r0 = gl * RPL;
    const int ng = (N + 2 * HC - 1) / (2 * HC);
    const bool active = grp < ng;
    const bool warp_active = (tid & ~31) / JL < ng;     // the warp's first group is active
    float xa[HC][RPL], xb[HC][RPL], na[HC], nb[HC];
#pragma unroll
    for (int j = 0; j < HC; ++j) {
        const int ca = grp * HC + j, cb = (grp + ng) * HC + j;
        const float *pa = (active && ca < N) ? (ca < k ? sC + ca * LDS : sB + (ca - k) * LDS) : nullptr;
        const float *pb = (active && cb < N) ? (cb < k ? sC + cb * LDS : sB + (cb - k) * LDS) : nullptr;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const int row = r0 + i;
            xa[j][i] = (pa != nullptr && row < n) ? pa[row] : 0.f;
            xb[j][i] = (pb != nullptr && row < n) ? pb[row] : 0.f;
        }
    }
    // ||Z||_F^2 (invariant under the rotations) sets the level below which a column is noise
    {
        float f = 0.f;
#pragma unroll
        for (int j = 0; j < HC; ++j)
#pragma unroll
            for (int i = 0; i < RPL; ++i) f = fmaf(xa[j][i], xa[j][i], fmaf(xb[j][i], xb[j][i], f));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
        if ((tid & 31) == 0) stage_n[tid >> 5] = f;
    }
    __syncthreads();                          // inputs consumed: the staging area is free
    float fro2 = 0.f;
#pragma unroll
    for (int w = 0; w < FW; ++w) fro2 += stage_n[w];
    const float floor2 = JACOBI_ZERO * fro2;
    __syncthreads();                          // the staged norms area is free again
    const int destA = grp == 0 ? 0 : (grp < ng - 1 ? grp + 1 : 2 * ng - 1);
    const int destB = grp == 0 ? 1 : ng + grp - 1;
    int sweeps = 0;
    bool converged = false;
    while (sweeps < JACOBI_MAX_SWEEPS) {
        ++sweeps;
        int rotated = 0;
        if (warp_active) {
#pragma unroll
            for (int j = 0; j < HC; ++j) {
                float sa = 0.f, sb = 0.f;
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    sa = fmaf(xa[j][i], xa[j][i], sa);
                    sb = fmaf(xb[j][i], xb[j][i], sb);
                }
                na[j] = group_sum(sa);
                nb[j] = group_sum(sb);
            }
        }
#pragma unroll 1
        for (int round = 0; round < 2 * ng - 1; ++round) {
            if (warp_active) {
                if (round == 0) {
#pragma unroll
                    for (int j1 = 0; j1 < HC; ++j1)
#pragma unroll
                        for (int j2 = j1 + 1; j2 < HC; ++j2) {
                            jrot<RPL>(xa[j1], xa[j2], na[j1], na[j2], floor2, rotated);
                            jrot<RPL>(xb[j1], xb[j2], nb[j1], nb[j2], floor2, rotated);
                        }
                }
                JCrossAll<HC, RPL, 0>::run(xa, xb, na, nb, floor2, rotated);
            }
            if (ng > 1) {                     // move the slots for the next round
                // two staging buffers, alternating by round: a round's writes never meet the
                // previous round's reads, so one barrier per round suffices
                float *stg = stage + (round & 1) * (2 * ng * HC * SS);
                float *stn = stage_n + (round & 1) * (2 * ng * HC);
                if (active) {
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        float *da = stg + (destA * HC + j) * SS + r0;
                        float *db = stg + (destB * HC + j) * SS + r0;
#pragma unroll
                        for (int i = 0; i < RPL; ++i) {
                            da[i] = xa[j][i];
                            db[i] = xb[j][i];
                        }
                        if (gl == 0) {
                            stn[destA * HC + j] = na[j];
                            stn[destB * HC + j] = nb[j];
                        }
                    }
                }
                __syncthreads();
                if (active) {
#pragma unroll
                    for (int j = 0; j < HC; ++j) {
                        const float *sa = stg + (grp * HC + j) * SS + r0;
                        const float *sb = stg + ((ng + grp) * HC + j) * SS + r0;
#pragma unroll
                        for (int i = 0; i < RPL; ++i) {
                            xa[j][i] = sa[i];
                            xb[j][i] = sb[i];
                        }
                        na[j] = stn[grp * HC + j];
                        nb[j] = stn[(ng + grp) * HC + j];
                    }
                }
            }
        }
        if (__syncthreads_or(rotated) == 0) {
            converged = true;
            break;
        }
    }
    // final columns (position order) and their exact norms
    if (warp_active) {
#pragma unroll
        for (int j = 0; j < HC; ++j) {
            float sa = 0.f, sb = 0.f;
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                sa = fmaf(xa[j][i], xa[j][i], sa);
                sb = fmaf(xb[j][i], xb[j][i], sb);
            }
            sa = group_sum(sa);
            sb = group_sum(sb);
            if (active) {
                float *da = stage + (grp * HC + j) * SS + r0;
                float *db = stage + ((ng + grp) * HC + j) * SS + r0;
#pragma unroll
                for (int i = 0; i < RPL; ++i) {
                    da[i] = xa[j][i];
                    db[i] = xb[j][i];
                }
                if (gl == 0) {
                    nrm_out[grp * HC + j] = sqrtf(sa);
                    nrm_out[(ng + grp) * HC + j] = sqrtf(sb);
                }
            }
        }
    }
    __syncthreads();
    return converged ? sweeps : -sweeps;
}

// Register-tiled product over shared-memory operands: out(i, j, sum_l A(i, l) B(l, j)) for
// i < M, j < N, l < K, each thread accumulating TI x TJ outputs (rows ib + MS ii, columns
// TJ jb + jj). Lanes of a warp take consecutive ib, so row-strided A loads fall in distinct banks
// (odd row stride) and B loads are shared by the lanes of a column block.
template <int TI, int TJ, class LA, class LB, class ST>
__device__ __forceinline__ void tile_gemm(int M, int N, int K, LA la, LB lb, ST st) {
    const int MS = (M + TI - 1) / TI, NSB = (N + TJ - 1) / TJ;
    for (int t = threadIdx.x; t < MS * NSB; t += FT) {
        const int ib = t % MS, jb = t / MS;
        int ii_[TI], jj_[TJ];
#pragma unroll
        for (int a = 0; a < TI; ++a) ii_[a] = min(ib + MS * a, M - 1);
#pragma unroll
        for (int b = 0; b < TJ; ++b) jj_[b] = min(TJ * jb + b, N - 1);
        float acc[TI][TJ];
#pragma unroll
        for (int a = 0; a < TI; ++a)
#pragma unroll
            for (int b = 0; b < TJ; ++b) acc[a][b] = 0.f;
#pragma unroll 2
        for (int l = 0; l < K; ++l) {
            float av[TI], bv[TJ];
#pragma unroll
            for (int a = 0; a < TI; ++a) av[a] = la(ii_[a], l);
#pragma unroll
            for (int b = 0; b < TJ; ++b) bv[b] = lb(l, jj_[b]);
#pragma unroll
            for (int a = 0; a < TI; ++a)
#pragma unroll
                for (int b = 0; b < TJ; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
        }
#pragma unroll
        for (int a = 0; a < TI; ++a)
#pragma unroll
            for (int b = 0; b < TJ; ++b) {
                const int i = ib + MS * a, j = TJ * jb + b;
                if (i < M && j < N) st(i, j, acc[a][b]);
            }
    }
}

// Householder QR in shared memory (R in place, reflectors kept below it).
//
// Step j reflects the pivot row j and the body rows y0(j) .. y1 - 1 of column j: lane l holds
// body rows y0 + l + 32 u (u < 4) of the reflector in registers. Warp 0 updates column j + 1
// alone and forms the next reflector from the updated values in its registers; warps 1 .. FW - 1
// update the other trailing columns, eight at a time with overlapped reductions. Each step
// therefore ends with a single barrier, and the next reflector is off the other warps' path.
// Reflectors are stored scaled in the body rows of their column (v_i below the pivot, v_pivot = 1
// implicit) with tau_j in sTau[j]; R's diagonal entries replace the pivots.
//
// Storage policies: element (i, c) of a body row is at(i, c); the pivot row of step j is the
// vector pivot(j) with stride pstride; body rows number at most 128.
struct CoreRows {               // the fold core Z: Sigma rows in sC, block rows in sY (row-major)
    float *sY, *sC;
    int k, b;
    __device__ float *pivot(int j) const { return j < k ? sC + j * LDS : sY + (j - k) * LDS; }
    __device__ int pstride() const { return 1; }
    __device__ int y0(int j) const { return j < k ? 0 : j - k + 1; }
    __device__ int y1() const { return b; }
    __device__ float &at(int i, int c) const { return sY[i * LDS + c]; }
};
struct ColumnRows {             // a D-row matrix stored by columns in sC (column c at sC + c LDS)
    float *sC;
    __device__ float *pivot(int j) const { return sC + j; }
    __device__ int pstride() const { return LDS; }
    __device__ int y0(int j) const { return j + 1; }
    __device__ int y1() const { return D; }
    __device__ float &at(int i, int c) const { return sC[c * LDS + i]; }
};

// Reflector of column j from its body values x[u] (rows y0 + lane + 32 u, those below `from`
// taking part) and the pivot entry `alpha`: stores v = x * scale below the pivot, beta at the
// pivot and tau. Called by one full warp.
template <class M>
__device__ __forceinline__ void qr_reflector(const M &m, int j, int y0, int from, float alpha,
                                             const float (&x)[4], float *sTau) {
    const int lane = threadIdx.x & 31, y1 = m.y1();
    float s2 = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = y0 + lane + 32 * u;
        if (i < y1 && i >= from) s2 = fmaf(x[u], x[u], s2);
    }
    s2 = warp_sum(s2);
    float tau = 0.f, beta = alpha, scale = 0.f;
    if (s2 > 0.f) {
        beta = -copysignf(sqrtf(fmaf(alpha, alpha, s2)), alpha);
        tau = (beta - alpha) / beta;
        scale = 1.f / (alpha - beta);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = y0 + lane + 32 * u;
        if (i < y1 && i >= from) m.at(i, j) = x[u] * scale;
    }
    __syncwarp();
    if (lane == 0) {
        m.pivot(j)[j * m.pstride()] = beta;
        sTau[j] = tau;
    }
}

template <class M>
__device__ void householder_qr(const M &m, int n, float *sTau) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ps = m.pstride(), y1 = m.y1();
    if (warp == 0 && n > 0) {                        // reflector of column 0
        const int y0 = m.y0(0);
        float x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = y0 + lane + 32 * u;
            x[u] = i < y1 ? m.at(i, 0) : 0.f;
        }
        qr_reflector(m, 0, y0, y0, m.pivot(0)[0], x, sTau);
    }
    __syncthreads();
    for (int j = 0; j < n; ++j) {
        const float tau = sTau[j];
        const int y0 = m.y0(j);
        const int y0n = j + 1 < n ? m.y0(j + 1) : y1;  // body of the next step
        float *pr = m.pivot(j);
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = y0 + lane + 32 * u;
            v[u] = i < y1 ? m.at(i, j) : 0.f;
        }
        if (warp == 0) {
            // column j + 1 alone, then its reflector (the next step's), off the other warps' path
            if (j + 1 < n) {
                const int c = j + 1;
                float x[4], w = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = y0 + lane + 32 * u;
                    x[u] = i < y1 ? m.at(i, c) : 0.f;
                    w = fmaf(v[u], x[u], w);
                }
                w = warp_sum(w);
                const float pj = pr[c * ps];
                const float wq = (w + pj) * tau;
                __syncwarp();
                if (lane == 0) pr[c * ps] = pj - wq;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = y0 + lane + 32 * u;
                    x[u] = fmaf(-wq, v[u], x[u]);
                    if (i < y1) m.at(i, c) = x[u];
                }
                // the next pivot: a body row of this step (one lane holds it) or untouched
                const int rel = y0n - 1 - y0;
                float al;
                if (rel >= 0) {
                    const int ur = rel >> 5;
                    const float cand = ur == 0 ? x[0] : ur == 1 ? x[1] : ur == 2 ? x[2] : x[3];
                    al = __shfl_sync(0xffffffffu, cand, rel & 31);
                } else {
                    al = m.pivot(j + 1)[(j + 1) * ps];
                }
                __syncwarp();
                qr_reflector(m, j + 1, y0, y0n, al, x, sTau);
            }
        } else {
            // columns j + 2 ... over warps 1 .. FW - 1, eight per batch (overlapped reductions)
            constexpr int W1 = FW - 1;
            for (int cb = j + 2 + (warp - 1); cb < n; cb += 8 * W1) {
                float w[8], xq[8][4], pj[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int c = min(cb + q * W1, n - 1);
                    w[q] = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = y0 + lane + 32 * u;
                        xq[q][u] = i < y1 ? m.at(i, c) : 0.f;
                        w[q] = fmaf(v[u], xq[q][u], w[q]);
                    }
                    pj[q] = pr[c * ps];
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                    for (int q = 0; q < 8; ++q) w[q] += __shfl_xor_sync(0xffffffffu, w[q], o);
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int c = cb + q * W1;
                    if (c < n) {
                        const float wq = (w[q] + pj[q]) * tau;
                        if (lane == 0) pr[c * ps] = pj[q] - wq;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int i = y0 + lane + 32 * u;
                            if (i < y1) m.at(i, c) = fmaf(-wq, v[u], xq[q][u]);
                        }
                    }
                }
                __syncwarp();
            }
        }
        __syncthreads();
    }
}

// Triangular factor of the core, in place: Z = Q R, keeping R only. R^T R = Z^T Z, so R has the
// singular values and the right singular vectors H of Z, and the one-sided Jacobi on the rows of
// R converges in fewer sweeps than on the rows of Z (triangular preconditioning of the Hestenes
// method). Z's rows are vectors of length n: row c < k (Sigma_c e_c) at sC + c LDS, row k + i (the
// block's [S | T] row i) at sY + i LDS; the Sigma rows are diagonal, so the reflector of column
// j < k involves only row j and the b block rows, and column j >= k pivots on block row j - k. On
// return R's row c is stored where Z's row c was, entries below the diagonal cleared (block rows
// p .. b - 1 become zero).
__device__ void core_triangular_factor(float *sY, float *sC, float *sTau, int k, int b, int n) {
    householder_qr(CoreRows{sY, sC, k, b}, n, sTau);
    for (int o = threadIdx.x; o < b * n; o += FT) {
        const int i = o / n, c = o % n;
        if (c < k + i) sY[i * LDS + c] = 0.f;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(FT, 1) fold_core_kernel(FoldArgs a) {
    extern __shared__ float smem[];
    float *sA = smem + OFF_A;
    float *sB = smem + OFF_B;
    float *sC = smem + OFF_C;
    float *sTau = smem + OFF_TAU;
    float *sSig = smem + OFF_SIG;
    float *sNrm = smem + OFF_NRM;
    float *sSN = smem + OFF_SNRM;
    float *sScr = smem + OFF_SCR;
    int *sSel = reinterpret_cast<int *>(smem + OFF_INT);
    float *stage = sB;                    // Jacobi staging overlays B and C

    const FoldPath P = (a.path_lo + (int)blockIdx.y) ? a.path[1] : a.path[0];
    const int unit = a.unit0 + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = P.k, r = P.r, p = P.p, kp = P.kp, b = a.b;
    const int n = k + p;                  // rows of Z^T (columns of Z)
    const size_t ring_base = (size_t)unit * a.R * D;
    const float *Bin = P.basis_in + (size_t)unit * D * r;

    // ---- load F (b x D) from the exact window ring, B (as k columns) and Sigma ---------------
    auto load_F = [&]() {
        if (a.kv_dtype == ISKV_BF16) {
            const __nv_bfloat16 *ring = reinterpret_cast<const __nv_bfloat16 *>(P.ring);
            const int nv = b * (D / 8);
            for (int v0 = tid; v0 < nv; v0 += 4 * FT) {
                uint4 u[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int v = v0 + q * FT;
                    if (v < nv) {
                        const int i = v >> 4, j8 = (v & 15) * 8;
                        const int slot = (a.slot0 + i) % a.R;
                        u[q] = *reinterpret_cast<const uint4 *>(ring + ring_base + (size_t)slot * D + j8);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int v = v0 + q * FT;
                    if (v < nv) {
                        const int i = v >> 4, j8 = (v & 15) * 8;
                        const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
                        float *dst = sA + i * LDS + j8;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            dst[2 * e] = __uint_as_float(w[e] << 16);
                            dst[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
                        }
                    }
                }
            }
        } else {
            const float *ring = reinterpret_cast<const float *>(P.ring);
            const int nv = b * (D / 4);
            for (int v0 = tid; v0 < nv; v0 += 4 * FT) {
                float4 u[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int v = v0 + q * FT;
                    if (v < nv) {
                        const int i = v >> 5, j4 = (v & 31) * 4;
                        const int slot = (a.slot0 + i) % a.R;
                        u[q] = *reinterpret_cast<const float4 *>(ring + ring_base + (size_t)slot * D + j4);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int v = v0 + q * FT;
                    if (v < nv) {
                        const int i = v >> 5, j4 = (v & 31) * 4;
                        float *dst = sA + i * LDS + j4;
                        dst[0] = u[q].x;
                        dst[1] = u[q].y;
                        dst[2] = u[q].z;
                        dst[3] = u[q].w;
                    }
                }
            }
        }
    };
    load_F();
    for (int o0 = tid; o0 < D * k; o0 += 4 * FT) {
        float v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int o = o0 + q * FT;
            v[q] = o < D * k ? Bin[(size_t)(o / k) * r + o % k] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int o = o0 + q * FT;
            if (o < D * k) sC[(o % k) * LDS + o / k] = v[q];
        }
    }
    if (tid < k) sSig[tid] = P.sigma_in[(size_t)unit * r + tid];
    __syncthreads();

    // ---- step 1: S = F B (into Y[:, :k]) and the residual E = F - S B^T (in place) -----------
    if (k > 0) {
        tile_gemm<2, 4>(b, k, D, [&](int i, int l) { return sA[i * LDS + l]; },
                        [&](int l, int c) { return sC[c * LDS + l]; },
                        [&](int i, int c, float v) { sB[i * LDS + c] = v; });
        __syncthreads();
        tile_gemm<2, 4>(b, D, k, [&](int i, int c) { return sB[i * LDS + c]; },
                        [&](int c, int j) { return sC[c * LDS + j]; },
                        [&](int i, int j, float v) { sA[i * LDS + j] -= v; });
        __syncthreads();
    }

    // ---- residual basis: Householder QR of [B, E^T(rows 0..p-1)] (D x n, columns in sC) ------
    for (int o = tid; o < p * D; o += FT) {
        const int i = o / D, j = o % D;
        sC[(k + i) * LDS + j] = sA[i * LDS + j];
    }
    __syncthreads();
    householder_qr(ColumnRows{sC}, n, sTau);

    // ---- T = F P for the rows in the QR: T[i][l] = R[k+l][k+i] (l <= i) ----------------------
    for (int o = tid; o < p * p; o += FT) {
        const int i = o / p, l = o % p;
        sB[i * LDS + k + l] = (l <= i) ? sC[(k + i) * LDS + k + l] : 0.f;
    }
    // ---- P = Q[:, k:k+p] into sA columns 0..p-1 (over E rows 0..p-1, no longer needed) -------
    //      warp w builds columns l = w + FW q, eight at a time (overlapped reductions)
    for (int lb = warp; lb < p; lb += 8 * FW) {
        float xr[8][4];
        int lmax = lb;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int l = lb + q * FW;
            if (l < p) lmax = l;
#pragma unroll
            for (int u = 0; u < 4; ++u) xr[q][u] = (lane + 32 * u == k + l) ? 1.f : 0.f;
        }
        for (int jc = min(n - 1, k + lmax); jc >= 0; --jc) {
            const float tau = sTau[jc];
            if (tau == 0.f) continue;
            const float *v = sC + jc * LDS;
            float vv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = lane + 32 * u;
                vv[u] = i > jc ? v[i] : (i == jc ? 1.f : 0.f);
            }
            float w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                w[q] = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) w[q] = fmaf(vv[u], xr[q][u], w[q]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q] += __shfl_xor_sync(0xffffffffu, w[q], o);
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int u = 0; u < 4; ++u) xr[q][u] = fmaf(-w[q] * tau, vv[u], xr[q][u]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int l = lb + q * FW;
            if (l < p)
#pragma unroll
                for (int u = 0; u < 4; ++u) sA[l * LDS + lane + 32 * u] = xr[q][u];
        }
    }
    __syncthreads();
    // ---- rows that did not enter the QR (p < b): T[i] = E[i] P ---------------------------------
    for (int o = tid; o < (b - p) * p; o += FT) {
        const int i = p + o / p, l = o % p;
        const float *e = sA + i * LDS, *pc = sA + l * LDS;
        float s0 = 0.f, s1 = 0.f;
        for (int j = 0; j < D; j += 2) {
            s0 = fmaf(e[j], pc[j], s0);
            s1 = fmaf(e[j + 1], pc[j + 1], s1);
        }
        sB[i * LDS + k + l] = s0 + s1;
    }
    // ---- Z^T columns 0..k-1: Sigma_c e_c (length n) -------------------------------------------
    for (int o = tid; o < k * n; o += FT) {
        const int c = o / n, m = o % n;
        sC[c * LDS + m] = (m == c) ? sSig[c] : 0.f;
    }
    __syncthreads();

    // ---- Z -> R (same Z^T Z), then one-sided Jacobi on the n columns of R^T, register resident
    core_triangular_factor(sB, sC, sTau, k, b, n);
    const int NJ = n;                     // Jacobi columns: the rows of R
    int sweeps;
    const int HC = NJ <= 96 ? 3 : 4;     // NJ = k + p <= D
    {
        const int rpl = n <= 96 ? 6 : (n <= 112 ? 7 : 8);
        switch (HC * 16 + rpl) {
            case 3 * 16 + 6: sweeps = jacobi_regs<3, 6>(sB, sC, k, NJ, n, stage, sSN, sNrm); break;
            case 3 * 16 + 7: sweeps = jacobi_regs<3, 7>(sB, sC, k, NJ, n, stage, sSN, sNrm); break;
            case 3 * 16 + 8: sweeps = jacobi_regs<3, 8>(sB, sC, k, NJ, n, stage, sSN, sNrm); break;
            case 4 * 16 + 6: sweeps = jacobi_regs<4, 6>(sB, sC, k, NJ, n, stage, sSN, sNrm); break;
            case 4 * 16 + 7: sweeps = jacobi_regs<4, 7>(sB, sC, k, NJ, n, stage, sSN, sNrm); break;
            default: sweeps = jacobi_regs<4, 8>(sB, sC, k, NJ, n, stage, sSN, sNrm); break;
        }
    }
    const int NC = 2 * ((NJ + 2 * HC - 1) / (2 * HC)) * HC;  // staged columns (NC - NJ zero)
    if (tid == 0) {
        if (sweeps < 0) set_status(a.status, ISKV_ERR_NOT_CONVERGED);
        if (a.stats) {
            const unsigned long long sw = (unsigned long long)(sweeps < 0 ? -sweeps : sweeps);
            atomicMax(a.stats, sw);
            atomicAdd(a.stats + 1, sw);
            atomicAdd(a.stats + 2, 1ull);
        }
    }

    // ---- singular values = column norms; select the top kp (descending, ties by index) -------
    for (int c = tid; c < NC; c += FT) {
        if (!isfinite(sNrm[c])) {
            set_status(a.status, ISKV_ERR_NONFINITE);
            sNrm[c] = -1.f;
        }
    }
    __syncthreads();
    // columns at or below the Jacobi's noise level (it leaves them unrotated) count as zero
    float zthr;
    {
        float f = 0.f;
        for (int c = lane; c < NC; c += 32) f = fmaf(fmaxf(sNrm[c], 0.f), fmaxf(sNrm[c], 0.f), f);
        zthr = sqrtf(JACOBI_ZERO * warp_sum(f));
    }
    for (int c = tid; c < NC; c += FT) {
        const float s = sNrm[c];
        int rank = 0;
        for (int c2 = 0; c2 < NC; ++c2) {
            const float s2 = sNrm[c2];
            rank += (s2 > s) || (s2 == s && c2 < c);
        }
        if (rank < kp) sSel[rank] = c;
    }
    __syncthreads();
    // normalise the selected columns in place: they become the columns of H (length n)
    for (int o = tid; o < kp * n; o += FT) {
        const int c = o / n, m = o % n;
        const int cs = sSel[c];
        const float s = sNrm[cs];
        if (s > zthr) stage[cs * SS + m] /= s;
    }
    __syncthreads();
    // exactly-zero singular values: complete H with orthonormal directions (rank-deficient input)
    if (warp == 0) {
        float *v = sScr;
        for (int c = 0; c < kp; ++c) {
            const int cs = sSel[c];
            if (sNrm[cs] > zthr) continue;
            float *x = stage + cs * SS;
            for (int e = 0; e < n; ++e) {
                for (int m = lane; m < n; m += 32) v[m] = (m == e) ? 1.f : 0.f;
                __syncwarp();
                for (int c2 = 0; c2 < kp; ++c2) {
                    const int cs2 = sSel[c2];
                    if (c2 == c || (sNrm[cs2] <= zthr && c2 > c)) continue;
                    const float *y = stage + cs2 * SS;
                    float d = 0.f;
                    for (int m = lane; m < n; m += 32) d = fmaf(y[m], v[m], d);
                    d = warp_sum(d);
                    for (int m = lane; m < n; m += 32) v[m] = fmaf(-d, y[m], v[m]);
                    __syncwarp();
                }
                float nn = 0.f;
                for (int m = lane; m < n; m += 32) nn = fmaf(v[m], v[m], nn);
                nn = warp_sum(nn);
                if (nn > 0.25f) {
                    const float inv = 1.f / sqrtf(nn);
                    for (int m = lane; m < n; m += 32) x[m] = v[m] * inv;
                    __syncwarp();
                    break;
                }
                __syncwarp();
            }
            if (lane == 0) sNrm[cs] = 0.f;
        }
    }
    // ---- W = [P | B_old] as columns of sA (B_old at columns p .. p+k-1) ------------------------
    for (int o0 = tid; o0 < D * k; o0 += 4 * FT) {
        float v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int o = o0 + q * FT;
            v[q] = o < D * k ? Bin[(size_t)(o / k) * r + o % k] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int o = o0 + q * FT;
            if (o < D * k) sA[(p + o % k) * LDS + o / k] = v[q];
        }
    }
    __syncthreads();
    // ---- sign convention: new basis vector c points along old basis vector c (H[c][c] >= 0) ----
    const int ksg = k < kp ? k : kp;
    for (int c = tid; c < ksg; c += FT) sTau[c] = stage[sSel[c] * SS + c] < 0.f ? -1.f : 1.f;
    __syncthreads();
    for (int o = tid; o < ksg * n; o += FT) {
        const int c = o / n, m = o % n;
        if (sTau[c] < 0.f) stage[sSel[c] * SS + m] = -stage[sSel[c] * SS + m];
    }
    __syncthreads();

    // ---- outputs: Sigma+, H_top, B+ = [B P] H ------------------------------------------------
    float *sig_out = P.sigma_out + (size_t)unit * r;
    for (int c = tid; c < r; c += FT) sig_out[c] = c < kp ? sNrm[sSel[c]] : 0.f;
    float *ht = P.htop + (size_t)unit * r * r;
    for (int o = tid; o < k * kp; o += FT) {
        const int l = o / kp, c = o % kp;
        ht[(size_t)l * r + c] = stage[sSel[c] * SS + l];
    }
    float *Bout = P.basis_out + (size_t)unit * D * r;
    // dense H rows in the order of W's columns: Hd[l][c] = H[k + l][c] (P part), H[l - p][c] (B)
    float *Hd = sC + 512;                  // past the staged columns (NC SS <= 128 LDS + 384)
    for (int o = tid; o < n * kp; o += FT) {
        const int l = o / kp, c = o % kp;
        Hd[o] = stage[sSel[c] * SS + (l < p ? k + l : l - p)];
    }
    __syncthreads();
    tile_gemm<4, 4>(D, kp, n, [&](int j, int l) { return sA[l * LDS + j]; },
                    [&](int l, int c) { return Hd[l * kp + c]; },
                    [&](int j, int c, float v) { Bout[(size_t)j * r + c] = v; });
    for (int o = tid; o < D * (r - kp); o += FT)
        Bout[(size_t)(o / (r - kp)) * r + kp + o % (r - kp)] = 0.f;
    __syncthreads();                       // H, W consumed; B+ (uncorrected) and H_top written
    // ---- one Newton-Schulz step towards the nearest orthonormal basis, B+ <- B+ (3I - M) / 2 with
    //      M = B+^T B+ (the Jacobi stops at a relative orthogonality threshold, and without this
    //      the loss of orthonormality would add up over folds); H_top gets the same right factor so
    //      old coordinates stay consistent with the corrected basis.
    float *sBp = sC;                       // B+ columns [kp][LDS]
    float *sM = sB;                        // M [kp][kp]
    float *sH = sA;                        // H_top [k][kp + 1]
    const int hld = kp + 1;
    for (int o = tid; o < D * kp; o += FT) sBp[(o % kp) * LDS + o / kp] = Bout[(size_t)(o / kp) * r + o % kp];
    for (int o = tid; o < k * kp; o += FT) sH[(o / kp) * hld + o % kp] = ht[(size_t)(o / kp) * r + o % kp];
    __syncthreads();
    tile_gemm<2, 4>(kp, kp, D, [&](int c, int j) { return sBp[c * LDS + j]; },
                    [&](int j, int c2) { return sBp[c2 * LDS + j]; },
                    [&](int c, int c2, float v) { sM[c * kp + c2] = v; });
    __syncthreads();
    tile_gemm<4, 4>(D, kp, kp, [&](int j, int c2) { return sBp[c2 * LDS + j]; },
                    [&](int c2, int c) { return sM[c2 * kp + c]; },
                    [&](int j, int c, float v) {
                        Bout[(size_t)j * r + c] = 1.5f * sBp[c * LDS + j] - 0.5f * v;
                    });
    tile_gemm<2, 4>(k, kp, kp, [&](int l, int c2) { return sH[l * hld + c2]; },
                    [&](int c2, int c) { return sM[c2 * kp + c]; },
                    [&](int l, int c, float v) {
                        ht[(size_t)l * r + c] = 1.5f * sH[l * hld + c] - 0.5f * v;
                    });
    __syncthreads();
    // corrected B+ columns back into shared memory; reload F for the new rows' coordinates
    for (int o = tid; o < D * kp; o += FT) sBp[(o % kp) * LDS + o / kp] = Bout[(size_t)(o / kp) * r + o % kp];
    load_F();
    __syncthreads();
    // ---- new rows' coordinates C[n_c + i] = F[i] B+ --------------------------------------------
    if (a.skip_new_rows) return;
    const size_t cn0 = ((size_t)unit * a.n_max + a.n_c) * r;
    tile_gemm<2, 4>(b, kp, D, [&](int i, int jj) { return sA[i * LDS + jj]; },
                    [&](int jj, int c) { return sBp[c * LDS + jj]; },
                    [&](int i, int c, float v) { store_coord(P.coords, cn0 + (size_t)i * r + c, v, a.cbf); });
    for (int o = tid; o < b * (r - kp); o += FT)
        store_coord(P.coords, cn0 + (size_t)(o / (r - kp)) * r + kp + o % (r - kp), 0.f, a.cbf);
}

// History rotation: old coordinates move with the basis, C[0:n] <- C[0:n] H[:k] (iS-KV summary,
// "Block-Incremental Decoding Updates", U+ = diag(U, I_b) G, so the old rows of U+ Sigma+ are
// U Sigma H[:k]). Stale mode keeps the old coordinates (zero-padded to the new rank).
constexpr int ROT_THREADS = 256;              // 16 row groups x 16 column groups
constexpr int ROT_GX = 24;                    // CTAs per (unit, path); each takes every 24th tile
constexpr int ROT_HS = 128;                   // stride of H_top in shared memory

// One tile: acc[rr][cc] = sum_l X[RPT rg + rr][l] H[l][CW cg + cc] (X^T and H in shared memory,
// transposed tile stride XS), stored to rows RPT rg + rr < rows, columns CW cg + cc < r of the
// coordinates. Each thread keeps an RPT x CW block of outputs in registers, so every shared-memory
// load feeds RPT or CW fused multiply-adds (packed in pairs of columns for even CW).
template <int CW, int RPT, int XS>
__device__ __forceinline__ void rot_tile(const float *sXt, const float *sH, int k, int rg, int cg,
                                         void *coords, size_t cu, long long row0, int rows, int r,
                                         int cbf) {
    float acc[RPT][CW];
    if constexpr ((CW & 1) == 0) {
        // even widths: H columns as float2 pairs, packed fused multiply-adds
        float2 a2[RPT][CW / 2];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int c2 = 0; c2 < CW / 2; ++c2) a2[rr][c2] = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int l = 0; l < k; ++l) {
            float xs[RPT];
#pragma unroll
            for (int q = 0; q < RPT / 4; ++q) {
                const float4 x = *reinterpret_cast<const float4 *>(sXt + l * XS + RPT * rg + 4 * q);
                xs[4 * q] = x.x;
                xs[4 * q + 1] = x.y;
                xs[4 * q + 2] = x.z;
                xs[4 * q + 3] = x.w;
            }
            float2 hv[CW / 2];
#pragma unroll
            for (int c2 = 0; c2 < CW / 2; ++c2)
                hv[c2] = *reinterpret_cast<const float2 *>(sH + l * ROT_HS + CW * cg + 2 * c2);
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                const float2 xx = make_float2(xs[rr], xs[rr]);
#pragma unroll
                for (int c2 = 0; c2 < CW / 2; ++c2) a2[rr][c2] = __ffma2_rn(xx, hv[c2], a2[rr][c2]);
            }
        }
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int c2 = 0; c2 < CW / 2; ++c2) {
                acc[rr][2 * c2] = a2[rr][c2].x;
                acc[rr][2 * c2 + 1] = a2[rr][c2].y;
            }
    } else {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int cc = 0; cc < CW; ++cc) acc[rr][cc] = 0.f;
#pragma unroll 4
        for (int l = 0; l < k; ++l) {
            float xs[RPT];
#pragma unroll
            for (int q = 0; q < RPT / 4; ++q) {
                const float4 x = *reinterpret_cast<const float4 *>(sXt + l * XS + RPT * rg + 4 * q);
                xs[4 * q] = x.x;
                xs[4 * q + 1] = x.y;
                xs[4 * q + 2] = x.z;
                xs[4 * q + 3] = x.w;
            }
            float hv[CW];
#pragma unroll
            for (int cc = 0; cc < CW; ++cc) hv[cc] = sH[l * ROT_HS + CW * cg + cc];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                for (int cc = 0; cc < CW; ++cc) acc[rr][cc] = fmaf(xs[rr], hv[cc], acc[rr][cc]);
        }
    }
    // rows RPT rg .. RPT rg + RPT - 1, columns CW cg .. ; the columns kp .. r - 1 are cleared by
    // the column groups past kp (their H columns are zero)
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) {
        const int i = RPT * rg + rr;
        if (i >= rows) continue;
        const size_t base = cu + (size_t)(row0 + i) * r;
#pragma unroll
        for (int cc = 0; cc < CW; ++cc) {
            const int c = CW * cg + cc;
            if (c < r) store_coord(coords, base + c, acc[rr][cc], cbf);
        }
    }
}

// RPT rows per thread, tiles of 16 RPT rows (64 or 128).
template <int RPT>
__global__ void __launch_bounds__(ROT_THREADS, 2) rotate_kernel(RotArgs a) {
    constexpr int ROWS = 16 * RPT;
    constexpr int XS = ROWS + 4;              // stride of the transposed row tile
    constexpr int LOGR = RPT == 8 ? 7 : 6;
    extern __shared__ float smem[];
    const RotPath P = (a.path_lo + (int)blockIdx.z) ? a.path[1] : a.path[0];
    const int unit = a.unit0 + blockIdx.y;
    const int k = P.k, kp = P.kp, r = P.r;
    const int tid = threadIdx.x;
    const long long tiles = (a.n_old + ROWS - 1) / ROWS;
    const size_t cu = (size_t)unit * a.n_max * r;
    if (a.stale) {
        // stale coordinates: kept as they are, columns k .. kp - 1 zero
        for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
            const long long row0 = t * ROWS;
            const int rows = (int)min((long long)ROWS, a.n_old - row0);
            for (int o = tid; o < rows * (r - k); o += ROT_THREADS) {
                const int i = o / (r - k), c = k + o % (r - k);
                store_coord(P.coords, cu + (size_t)(row0 + i) * r + c, 0.f, a.cbf);
            }
        }
        return;
    }
    float *sH = smem;                         // [k][ROT_HS], zero past kp
    float *sXt = sH + k * ROT_HS;             // [k][XS]: column l of the row tile
    const float *ht = P.htop + (size_t)unit * r * r;
    for (int o = tid; o < k * ROT_HS; o += ROT_THREADS) {
        const int l = o / ROT_HS, c = o % ROT_HS;
        sH[o] = c < kp ? ht[(size_t)l * r + c] : 0.f;
    }
    const int rg = tid >> 4, cg = tid & 15;
    const int cw = (kp + 15) >> 4;            // columns per thread (1 .. 8)
    // fp32 coordinates in 16-byte quads: the next tile's rows are loaded into registers while
    // this tile is computed (thread: row i = o mod ROWS of quad q = o / ROWS for o = tid + 256 s)
    const bool vec = !a.cbf && (k & 3) == 0 && (r & 3) == 0;
    const int nq = vec ? (ROWS * (k >> 2) + ROT_THREADS - 1) / ROT_THREADS : 0;   // <= 8
    float4 pre[8];
    auto prefetch = [&](long long t) {
        const long long row0 = t * ROWS;
        const int rows = (int)min((long long)ROWS, a.n_old - row0);
        const float *cf = static_cast<const float *>(P.coords) + cu;
#pragma unroll
        for (int sq = 0; sq < 8; ++sq) {
            const int o = tid + ROT_THREADS * sq, i = o & (ROWS - 1), q = o >> LOGR;
            pre[sq] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (sq < nq && 4 * q < k && i < rows)
                pre[sq] = *reinterpret_cast<const float4 *>(cf + (size_t)(row0 + i) * r + 4 * q);
        }
    };
    if (vec && blockIdx.x < tiles) prefetch(blockIdx.x);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const long long row0 = t * ROWS;
        const int rows = (int)min((long long)ROWS, a.n_old - row0);
        __syncthreads();                      // previous tile's reads of sXt are done
        if (vec) {
            // transposed store of the prefetched rows (consecutive threads: consecutive rows)
#pragma unroll
            for (int sq = 0; sq < 8; ++sq) {
                const int o = tid + ROT_THREADS * sq, i = o & (ROWS - 1), q = o >> LOGR;
                if (sq < nq && 4 * q < k) {
                    sXt[(4 * q + 0) * XS + i] = pre[sq].x;
                    sXt[(4 * q + 1) * XS + i] = pre[sq].y;
                    sXt[(4 * q + 2) * XS + i] = pre[sq].z;
                    sXt[(4 * q + 3) * XS + i] = pre[sq].w;
                }
            }
        } else {
            for (int o = tid; o < ROWS * k; o += ROT_THREADS) {
                const int i = o / k, l = o % k;
                sXt[l * XS + i] = i < rows ? load_coord(P.coords, cu + (size_t)(row0 + i) * r + l, a.cbf) : 0.f;
            }
        }
        __syncthreads();
        if (vec && t + gridDim.x < tiles) prefetch(t + gridDim.x);
        // (the 8-row variant runs only with kp <= 64: at most 4 columns per thread)
        switch (cw) {
            case 1: rot_tile<1, RPT, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
            case 2: rot_tile<2, RPT, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
            case 3: rot_tile<3, RPT, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
            case 4: rot_tile<4, RPT, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
            default:
                if constexpr (RPT == 4) {
                    switch (cw) {
                        case 5: rot_tile<5, 4, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
                        case 6: rot_tile<6, 4, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
                        case 7: rot_tile<7, 4, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
                        default: rot_tile<8, 4, XS>(sXt, sH, k, rg, cg, P.coords, cu, row0, rows, r, a.cbf); break;
                    }
                }
                break;
        }
        // columns past 16 cw (only when kp < r and 16 cw < r): zero
        if (16 * cw < r) {
            for (int o = tid; o < rows * r; o += ROT_THREADS) {
                const int i = o / r, c = o % r;
                if (c >= 16 * cw) store_coord(P.coords, cu + (size_t)(row0 + i) * r + c, 0.f, a.cbf);
            }
        }
    }
}

cudaError_t launch_fold(const FoldArgs &a, int n_units, cudaStream_t s) {
    if (a.path_hi <= a.path_lo || n_units <= 0) return cudaSuccess;
    static size_t attr[64] = {0};
    const size_t smem = fold_smem_bytes();
    const cudaError_t e = ensure_smem((const void *)fold_core_kernel, smem, attr);
    if (e != cudaSuccess) return e;
    fold_core_kernel<<<dim3(n_units, a.path_hi - a.path_lo), FT, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_rotate(const RotArgs &a, int n_units, cudaStream_t s) {
    if (a.n_old <= 0 || a.path_hi <= a.path_lo || n_units <= 0) return cudaSuccess;
    int kmax = 0, kpmax = 0;
    bool quads = !a.cbf;
    for (int x = a.path_lo; x < a.path_hi; ++x) {
        kmax = a.path[x].k > kmax ? a.path[x].k : kmax;
        kpmax = a.path[x].kp > kpmax ? a.path[x].kp : kpmax;
        quads = quads && (a.path[x].k & 3) == 0 && (a.path[x].r & 3) == 0;
    }
    // 8 rows per thread (128-row tiles) where the prefetch registers allow it (k <= 64) and the
    // output block stays small (kp <= 64); else 4 rows per thread (64-row tiles)
    const bool wide = quads && kmax <= 64 && kpmax <= 64;
    const int rows = wide ? 128 : 64;
    const size_t smem = (size_t)kmax * (ROT_HS + rows + 4) * sizeof(float) + 16;
    const long long tiles = (a.n_old + rows - 1) / rows;
    const long long gx = tiles < ROT_GX ? tiles : ROT_GX;
    const dim3 grid((unsigned)gx, n_units, a.path_hi - a.path_lo);
    if (wide) {
        static size_t attr[64] = {0};
        const cudaError_t e = ensure_smem((const void *)rotate_kernel<8>, smem, attr);
        if (e != cudaSuccess) return e;
        rotate_kernel<8><<<grid, ROT_THREADS, smem, s>>>(a);
    } else {
        static size_t attr[64] = {0};
        const cudaError_t e = ensure_smem((const void *)rotate_kernel<4>, smem, attr);
        if (e != cudaSuccess) return e;
        rotate_kernel<4><<<grid, ROT_THREADS, smem, s>>>(a);
    }
    return cudaGetLastError();
}

// ---- joint per-layer factorisation --------------------------------------------------------------
// All kv-heads of a (layer, sequence) share one factorisation over rows of length d = H D (the
// kv-heads' rows side by side). The fold of such a unit reduces to the per-head fold above through
// a change of coordinates: with k + b <= 128, the basis B (d x k) and the residual basis P (d x b)
// span at most 128 dimensions, and in the coordinates of [B P] the block is
// F~ = F [B P] = [F B | F P], the old basis is [I_k; 0] and the core Z, its SVD, H_top and the new
// rows' coordinates are exactly those of the d-dimensional fold ("Block-Incremental Decoding
// Updates", steps 1-3). So a joint fold is
//   1. joint_prep_kernel: S = F B over the kv-heads' slices, E = F - S B^T, and a Householder QR
//      of A = [B, E^T] (d x n, n = k + b) streamed over the kv-heads: the first head's 128 rows are
//      factorised directly, every later head's rows together with the triangular factor so far
//      (tall-skinny QR, one 128-row block per step). With A = [Q1 Q2] [[R11, R12], [0, R22]],
//      P = Q2, F P = R22^T (Q2 is orthogonal to B = Q1 R11 and to E's part along Q1) and
//      F B = S + R12^T R11 (what the single projection left along B). Writes F~ as a fp32 pseudo-
//      block of b rows of 128 and the pseudo-basis [I_k; 0]; keeps every step's Householder vectors;
//   2. fold_core_kernel on the pseudo-blocks (Sigma+, H_top, the basis B~+ in the coordinates of
//      [B P], the new rows' coordinates F~ B~+ = F B+);
//   3. joint_basis_kernel: B+ = [B P] B~+, forming each kv-head's 128 rows of P from the stored
//      Householder vectors (last head first: the rows of head h are the head's Householder
//      product applied to [W; 0], W the product of the later heads' top blocks).
// Both kernels: one CTA (256 threads) per joint unit and path (blockIdx.y = path).

// A 128-row matrix stored by rows (element (i, c) at s[i LDS + c]) whose pivot rows are its own
// rows: the first kv-head's QR step.
struct RowMajorRows {
    float *s;
    __device__ float *pivot(int j) const { return s + j * LDS; }
    __device__ int pstride() const { return 1; }
    __device__ int y0(int j) const { return j + 1; }
    __device__ int y1() const { return D; }
    __device__ float &at(int i, int c) const { return s[i * LDS + c]; }
};

size_t joint_prep_smem(int k, int b) {
    return ((size_t)2 * D * LDS + D + (size_t)b * (k + 1)) * sizeof(float);
}

__global__ void __launch_bounds__(FT, 1) joint_prep_kernel(JointArgs a) {
    extern __shared__ float smem[];
    const JointPath P = (a.path_lo + (int)blockIdx.y) ? a.path[1] : a.path[0];
    float *sY = smem;                      // [D][LDS] a kv-head's rows of A: [B_h | E_h^T]
    float *sR = sY + D * LDS;              // [n][LDS] triangular factor of the rows so far
    float *sTau = sR + D * LDS;            // [D]
    float *sS = sTau + D;                  // [b][k + 1] S = F B
    const int j = a.junit0 + blockIdx.x;
    const int k = P.k, b = a.b, n = k + b, H = a.H, r = P.r, ks = k + 1;
    const int tid = threadIdx.x;

    // kv-head h's rows of [B, F^T]: basis rows in columns 0 .. k-1, block rows transposed in
    // columns k .. n-1 (row i of sY is channel i of the head)
    auto stage = [&](int h) {
        const size_t u = (size_t)j * H + h;
        const float *Bh = P.basis_in + u * D * r;
        for (int o = tid; o < D * k; o += FT) {
            const int i = o / k, l = o % k;
            sY[i * LDS + l] = Bh[(size_t)i * r + l];
        }
        for (int o = tid; o < b * D; o += FT) {
            const int c = o / D, i = o % D;
            const int slot = (a.slot0 + c) % a.R;
            sY[i * LDS + k + c] = load_row_elem(P.ring, (u * a.R + slot) * D + i, a.kv_dtype);
        }
    };

    // ---- S = F B = sum_h F_h B_h ------------------------------------------------------------
    for (int o = tid; o < b * ks; o += FT) sS[o] = 0.f;
    if (k > 0) {
        for (int h = 0; h < H; ++h) {
            __syncthreads();
            stage(h);
            __syncthreads();
            tile_gemm<2, 4>(b, k, D, [&](int c, int i) { return sY[i * LDS + k + c]; },
                            [&](int i, int l) { return sY[i * LDS + l]; },
                            [&](int c, int l, float v) { sS[c * ks + l] += v; });
        }
    }
    // ---- per kv-head: E_h = F_h - S B_h^T, then one step of the tall-skinny QR of [B, E^T] ----
    for (int h = 0; h < H; ++h) {
        __syncthreads();
        stage(h);
        __syncthreads();
        for (int o = tid; o < D * b; o += FT) {
            const int i = o / b, c = o % b;
            float v = sY[i * LDS + k + c];
            for (int l = 0; l < k; ++l) v = fmaf(-sS[c * ks + l], sY[i * LDS + l], v);
            sY[i * LDS + k + c] = v;
        }
        __syncthreads();
        if (h == 0) {
            householder_qr(RowMajorRows{sY}, n, sTau);
            for (int o = tid; o < n * n; o += FT) {
                const int i = o / n, c = o % n;
                sR[i * LDS + c] = c >= i ? sY[i * LDS + c] : 0.f;
            }
        } else {
            // pivot rows: the triangular factor so far; body: this head's 128 rows
            householder_qr(CoreRows{sY, sR, n, D}, n, sTau);
        }
        float *rf = P.refl + ((size_t)j * H + h) * D * a.ldr;
        for (int o = tid; o < D * n; o += FT) {
            const int i = o / n, c = o % n;
            rf[(size_t)i * a.ldr + c] = sY[i * LDS + c];
        }
        for (int c = tid; c < n; c += FT) P.tau[((size_t)j * H + h) * a.ldr + c] = sTau[c];
    }
    __syncthreads();
    // ---- F B = S + R12^T R11 -------------------------------------------------------------------
    for (int o = tid; o < b * k; o += FT) {
        const int c = o / k, l = o % k;
        float v = 0.f;
        for (int m = 0; m <= l; ++m) v = fmaf(sR[m * LDS + k + c], sR[m * LDS + l], v);
        sS[c * ks + l] += v;
    }
    __syncthreads();
    // ---- pseudo-block [F B | R22^T | 0] and pseudo-basis [I_k; 0] ------------------------------
    float *blk = P.blk + (size_t)j * b * D;
    for (int o = tid; o < b * D; o += FT) {
        const int i = o / D, c = o % D;
        float v = 0.f;
        if (c < k) v = sS[i * ks + c];
        else if (c < n && c - k <= i) v = sR[c * LDS + k + i];   // R22[c - k][i]
        blk[o] = v;
    }
    float *pb = P.pbasis + (size_t)j * D * r;
    for (int o = tid; o < D * r; o += FT) {
        const int i = o / r, c = o % r;
        pb[o] = (i == c && c < k) ? 1.f : 0.f;
    }
}

size_t joint_basis_smem(int n, int b, int kp) {
    return ((size_t)D * (LDS + 1) + (size_t)n * (b + 1) + (size_t)n * kp + D) * sizeof(float);
}

// QB: columns of P per warp (b <= 8 QB)
template <int QB>
__global__ void __launch_bounds__(FT, 1) joint_basis_kernel(JointArgs a) {
    extern __shared__ float smem[];
    const JointPath P = (a.path_lo + (int)blockIdx.y) ? a.path[1] : a.path[0];
    const int j = a.junit0 + blockIdx.x;
    const int k = P.k, b = a.b, n = k + b, H = a.H, r = P.r, kp = P.kp;
    const int lw = b + 1, lb = k + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *sY = smem;                      // [D][LDS] one head's Householder vectors; then P_h, B_h
    float *sW = sY + D * (LDS + 1);        // [n][b + 1] W: the later heads' top blocks times [0; I_b]
    float *sBp = sW + n * lw;              // [n][kp] B~+ rows 0 .. n-1 (rows n .. 127 are zero)
    float *sTau = sBp + n * kp;            // [D]
    for (int o = tid; o < n * b; o += FT) {
        const int i = o / b, c = o % b;
        sW[i * lw + c] = (i == k + c) ? 1.f : 0.f;
    }
    const float *bo = P.pbasis_out + (size_t)j * D * r;
    for (int o = tid; o < n * kp; o += FT) sBp[o] = bo[(size_t)(o / kp) * r + o % kp];
    for (int h = H - 1; h >= 0; --h) {
        const float *rf = P.refl + ((size_t)j * H + h) * D * a.ldr;
        __syncthreads();                   // the previous head's P_h and B_h are consumed
        for (int o = tid; o < D * n; o += FT) sY[(o / n) * LDS + o % n] = rf[(size_t)(o / n) * a.ldr + o % n];
        for (int c = tid; c < n; c += FT) sTau[c] = P.tau[((size_t)j * H + h) * a.ldr + c];
        __syncthreads();
        // X = [W; 0] (head 0: its 128 rows hold W on top), warp w owning columns w + 8 q, lane l
        // rows l + 32 u; the head's reflectors applied last to first
        float xb[QB][4];
#pragma unroll
        for (int q = 0; q < QB; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = warp + FW * q, i = lane + 32 * u;
                xb[q][u] = (h == 0 && c < b && i < n) ? sW[i * lw + c] : 0.f;
            }
        for (int jr = n - 1; jr >= 0; --jr) {
            const float tau = sTau[jr];
            if (tau == 0.f) continue;
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = lane + 32 * u;
                const float y = sY[i * LDS + jr];
                // later heads: pivot in the top block (row jr of W), all 128 rows in the body;
                // head 0: unit pivot at row jr, vector below it
                v[u] = h > 0 ? y : (i > jr ? y : (i == jr ? 1.f : 0.f));
            }
            float w[QB], top[QB];
#pragma unroll
            for (int q = 0; q < QB; ++q) {
                w[q] = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) w[q] = fmaf(v[u], xb[q][u], w[q]);
                const int c = warp + FW * q;
                top[q] = (h > 0 && c < b) ? sW[jr * lw + c] : 0.f;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int q = 0; q < QB; ++q) w[q] += __shfl_xor_sync(0xffffffffu, w[q], o);
            __syncwarp();                  // every lane has read its top entries
#pragma unroll
            for (int q = 0; q < QB; ++q) {
                const int c = warp + FW * q;
                if (c < b) {
                    const float wq = (w[q] + top[q]) * tau;
                    if (h > 0 && lane == 0) sW[jr * lw + c] = top[q] - wq;
#pragma unroll
                    for (int u = 0; u < 4; ++u) xb[q][u] = fmaf(-wq, v[u], xb[q][u]);
                }
            }
            __syncwarp();
        }
        __syncthreads();                   // every warp is done with the Householder vectors
        float *sP = sY;                    // [D][b + 1] this head's rows of P
        float *sBh = sY + D * lw;          // [D][k + 1] this head's rows of B
#pragma unroll
        for (int q = 0; q < QB; ++q)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = warp + FW * q;
                if (c < b) sP[(lane + 32 * u) * lw + c] = xb[q][u];
            }
        const size_t uh = (size_t)j * H + h;
        const float *Bh = P.basis_in + uh * D * r;
        for (int o = tid; o < D * k; o += FT) sBh[(o / k) * lb + o % k] = Bh[(size_t)(o / k) * r + o % k];
        __syncthreads();
        float *Bo = P.basis_out + uh * D * r;
        tile_gemm<4, 4>(D, kp, n,
                        [&](int i, int l) { return l < k ? sBh[i * lb + l] : sP[i * lw + l - k]; },
                        [&](int l, int c) { return sBp[l * kp + c]; },
                        [&](int i, int c, float v) { Bo[(size_t)i * r + c] = v; });
        for (int o = tid; o < D * (r - kp); o += FT)
            Bo[(size_t)(o / (r - kp)) * r + kp + o % (r - kp)] = 0.f;
    }
}

cudaError_t launch_joint_prep(const JointArgs &a, int n_junits, cudaStream_t s) {
    if (a.path_hi <= a.path_lo || n_junits <= 0) return cudaSuccess;
    size_t smem = 0;
    for (int x = a.path_lo; x < a.path_hi; ++x) {
        const size_t v = joint_prep_smem(a.path[x].k, a.b);
        smem = v > smem ? v : smem;
    }
    static size_t attr[64] = {0};
    const cudaError_t e = ensure_smem((const void *)joint_prep_kernel, smem, attr);
    if (e != cudaSuccess) return e;
    joint_prep_kernel<<<dim3(n_junits, a.path_hi - a.path_lo), FT, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_joint_basis(const JointArgs &a, int n_junits, cudaStream_t s) {
    if (a.path_hi <= a.path_lo || n_junits <= 0) return cudaSuccess;
    size_t smem = 0;
    for (int x = a.path_lo; x < a.path_hi; ++x) {
        const size_t v = joint_basis_smem(a.path[x].k + a.b, a.b, a.path[x].kp);
        smem = v > smem ? v : smem;
    }
    const dim3 grid(n_junits, a.path_hi - a.path_lo);
    if (a.b <= 8 * 8) {
        static size_t attr[64] = {0};
        const cudaError_t e = ensure_smem((const void *)joint_basis_kernel<8>, smem, attr);
        if (e != cudaSuccess) return e;
        joint_basis_kernel<8><<<grid, FT, smem, s>>>(a);
    } else {
        static size_t attr[64] = {0};
        const cudaError_t e = ensure_smem((const void *)joint_basis_kernel<16>, smem, attr);
        if (e != cudaSuccess) return e;
        joint_basis_kernel<16><<<grid, FT, smem, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace iskv
