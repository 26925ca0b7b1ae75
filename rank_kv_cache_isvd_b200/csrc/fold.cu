// Block-incremental truncated-SVD update ("fold") of one (layer, sequence, kv-head, path) unit.
//
// iS-KV summary, "Block-Incremental Decoding Updates", steps 1-3, for history A = U Sigma B^T
// (k components, coordinates C = U Sigma stored) and pending block F (b rows of the window):
//   1. S = F B, E = F - S B^T (projected twice); orthonormal residual basis P (d x p) from a
//      Householder QR of [B, E^T] (its columns after the first k), p = min(b, d - k);
//   2. Z = [[Sigma, 0], [S, F P]], (k + b) x (k + p); with P from that QR, F P = E P is the
//      transpose of the QR's trailing R block for the rows that entered it;
//   3. (G, Sigma+, H) = SVD_r(Z) by one-sided (Hestenes) Jacobi on the columns of Z^T: at
//      convergence the columns of Z^T J are orthogonal, their norms are the singular values and
//      the normalised columns are the right singular vectors H of Z, so J is never accumulated;
//      B+ = [B P] H, the old coordinates move by H[:k] (kernel rotate_kernel) and the new rows'
//      coordinates are F B+ (bottom block of U+ Sigma+, since Z H = G Sigma+).
// One CTA per unit and path (blockIdx.y = path), everything in shared memory (b <= 128).
#include "iskv_internal.cuh"

namespace iskv {

constexpr int FOLD_THREADS = 512;
constexpr int FOLD_WARPS = FOLD_THREADS / 32;
constexpr int JG = 8;                         // lanes per Jacobi pair group
constexpr int JGROUPS = FOLD_THREADS / JG;    // pair groups per CTA
constexpr float JACOBI_TOL = 4e-6f;           // rotate while |a.b| > tol |a| |b|

size_t fold_smem_bytes() {
    return (size_t)(3 * 128 * LDS + 128 + 128 + 256 + FOLD_WARPS * 128) * sizeof(float) +
           (size_t)(128 + 4) * sizeof(int);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Round-robin (circle) schedule over Np players: in each of the Np - 1 rounds every player meets
// one other; over a sweep every pair meets once.
__device__ __forceinline__ void rr_pair(int Np, int round, int i, int &a, int &b) {
    const int M = Np - 1;
    if (i == 0) {
        a = 0;
        b = 1 + round % M;
    } else {
        a = 1 + (round + i) % M;
        b = 1 + (round - i + M) % M;
    }
}

__global__ void __launch_bounds__(FOLD_THREADS, 1) fold_core_kernel(FoldArgs a) {
    extern __shared__ float smem[];
    float *sA = smem;                    // F/E rows -> [P | B_old] columns -> F rows
    float *sB = sA + 128 * LDS;          // Y = [S | T] rows = Z^T columns k .. k+b-1
    float *sC = sB + 128 * LDS;          // QR columns -> Z^T columns 0 .. k-1 -> B+ columns
    float *sTau = sC + 128 * LDS;        // Householder tau
    float *sSig = sTau + 128;            // Sigma (old)
    float *sNrm = sSig + 128;            // column norms of Z^T J (up to 256 columns)
    float *sScr = sNrm + 256;            // per-warp scratch (128 floats each)
    int *sSel = reinterpret_cast<int *>(sScr + FOLD_WARPS * 128);
    int *sFlag = sSel + 128;

    const FoldPath P = blockIdx.y ? a.path[1] : a.path[0];
    const int unit = a.unit0 + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = P.k, r = P.r, p = P.p, kp = P.kp, b = a.b;
    const int n = k + p;                 // rows of Z^T (columns of Z)
    const int N = k + b;                 // columns of Z^T

    const size_t ring_base = (size_t)unit * a.R * D;
    const float *Bin = P.basis_in + (size_t)unit * D * r;

    // ---- load F (b x D) and B (as k columns), Sigma ------------------------------------------
    for (int o = tid; o < b * D; o += FOLD_THREADS) {
        const int i = o / D, j = o % D;
        const int slot = (a.slot0 + i) % a.R;
        sA[i * LDS + j] = load_row_elem(P.ring, ring_base + (size_t)slot * D + j, a.kv_dtype);
    }
    for (int o = tid; o < D * k; o += FOLD_THREADS) {
        const int j = o / k, c = o % k;
        sC[c * LDS + j] = Bin[(size_t)j * r + c];
    }
    if (tid < k) sSig[tid] = P.sigma[(size_t)unit * r + tid];
    if (tid == 0) sFlag[1] = 0;
    __syncthreads();

    // ---- step 1: S = F B (into Y[:, :k]); E = F - S B^T, twice (one warp per row) -------------
    if (k > 0) {
        float *scr = sScr + warp * 128;
        for (int i = warp; i < b; i += FOLD_WARPS) {
            float *f = sA + i * LDS;
            for (int c = lane; c < k; c += 32) {
                const float *bc = sC + c * LDS;
                float s = 0.f;
                for (int j = 0; j < D; ++j) s = fmaf(f[j], bc[j], s);
                sB[i * LDS + c] = s;
                scr[c] = s;
            }
            __syncwarp();
            for (int pass = 0; pass < 2; ++pass) {
                for (int j = lane; j < D; j += 32) {
                    float e = f[j];
                    for (int c = 0; c < k; ++c) e = fmaf(-scr[c], sC[c * LDS + j], e);
                    f[j] = e;
                }
                __syncwarp();
                if (pass == 0) {
                    for (int c = lane; c < k; c += 32) {
                        const float *bc = sC + c * LDS;
                        float s = 0.f;
                        for (int j = 0; j < D; ++j) s = fmaf(f[j], bc[j], s);
                        scr[c] = s;
                    }
                    __syncwarp();
                }
            }
        }
    }
    __syncthreads();

    // ---- residual basis: Householder QR of [B, E^T(rows 0..p-1)] (D x n, columns in sC) ------
    for (int o = tid; o < p * D; o += FOLD_THREADS) {
        const int i = o / D, j = o % D;
        sC[(k + i) * LDS + j] = sA[i * LDS + j];
    }
    __syncthreads();
    for (int jc = 0; jc < n; ++jc) {
        float *col = sC + jc * LDS;
        if (warp == 0) {
            float s2 = 0.f;
            for (int i = jc + 1 + lane; i < D; i += 32) s2 = fmaf(col[i], col[i], s2);
            s2 = warp_sum(s2);
            const float alpha = col[jc];
            float tau = 0.f, beta = alpha, scale = 0.f;
            if (s2 > 0.f) {
                beta = -copysignf(sqrtf(fmaf(alpha, alpha, s2)), alpha);
                tau = (beta - alpha) / beta;
                scale = 1.f / (alpha - beta);
            }
            __syncwarp();
            for (int i = jc + 1 + lane; i < D; i += 32) col[i] *= scale;
            if (lane == 0) {
                col[jc] = beta;
                sTau[jc] = tau;
            }
        }
        __syncthreads();
        const float tau = sTau[jc];
        if (tau != 0.f) {
            for (int c = jc + 1 + warp; c < n; c += FOLD_WARPS) {
                float *x = sC + c * LDS;
                float w = 0.f;
                for (int i = jc + 1 + lane; i < D; i += 32) w = fmaf(col[i], x[i], w);
                w = (warp_sum(w) + x[jc]) * tau;
                __syncwarp();
                if (lane == 0) x[jc] -= w;
                for (int i = jc + 1 + lane; i < D; i += 32) x[i] = fmaf(-w, col[i], x[i]);
            }
        }
        __syncthreads();
    }

    // ---- T = F P for the rows in the QR: T[i][l] = R[k+l][k+i] (l <= i) ----------------------
    for (int o = tid; o < p * p; o += FOLD_THREADS) {
        const int i = o / p, l = o % p;
        sB[i * LDS + k + l] = (l <= i) ? sC[(k + i) * LDS + k + l] : 0.f;
    }
    // ---- P = Q[:, k:k+p] into sA columns 0..p-1 (over E rows 0..p-1, no longer needed) -------
    for (int l = warp; l < p; l += FOLD_WARPS) {
        float *x = sA + l * LDS;
        for (int i = lane; i < D; i += 32) x[i] = (i == k + l) ? 1.f : 0.f;
        __syncwarp();
        for (int jc = min(n - 1, k + l); jc >= 0; --jc) {
            const float tau = sTau[jc];
            if (tau == 0.f) continue;
            const float *v = sC + jc * LDS;
            float w = 0.f;
            for (int i = jc + 1 + lane; i < D; i += 32) w = fmaf(v[i], x[i], w);
            w = (warp_sum(w) + x[jc]) * tau;
            __syncwarp();
            if (lane == 0) x[jc] -= w;
            for (int i = jc + 1 + lane; i < D; i += 32) x[i] = fmaf(-w, v[i], x[i]);
            __syncwarp();
        }
    }
    __syncthreads();
    // ---- rows that did not enter the QR (p < b): T[i] = E[i] P ---------------------------------
    for (int o = tid; o < (b - p) * p; o += FOLD_THREADS) {
        const int i = p + o / p, l = o % p;
        const float *e = sA + i * LDS, *pc = sA + l * LDS;
        float s = 0.f;
        for (int j = 0; j < D; ++j) s = fmaf(e[j], pc[j], s);
        sB[i * LDS + k + l] = s;
    }
    // ---- Z^T columns 0..k-1: Sigma_c e_c (length n) -------------------------------------------
    for (int o = tid; o < k * n; o += FOLD_THREADS) {
        const int c = o / n, m = o % n;
        sC[c * LDS + m] = (m == c) ? sSig[c] : 0.f;
    }
    __syncthreads();

    // ---- one-sided Jacobi on the N columns (length n) of Z^T ----------------------------------
    {
        const int Np = N + (N & 1);
        const int gid = tid / JG, gl = tid % JG;
        const unsigned gmask = 0xffu << ((lane / JG) * JG);
        bool converged = false;
        int sweeps = 0;
        for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS; ++sweep) {
            ++sweeps;
            if (tid == 0) sFlag[0] = 0;
            __syncthreads();
            for (int round = 0; round < Np - 1; ++round) {
                for (int i = gid; i < Np / 2; i += JGROUPS) {
                    int ca, cb;
                    rr_pair(Np, round, i, ca, cb);
                    if (ca >= N || cb >= N) continue;
                    float *xa = ca < k ? sC + ca * LDS : sB + (ca - k) * LDS;
                    float *xb = cb < k ? sC + cb * LDS : sB + (cb - k) * LDS;
                    float al = 0.f, be = 0.f, ga = 0.f;
                    for (int m = gl; m < n; m += JG) {
                        const float u = xa[m], v = xb[m];
                        al = fmaf(u, u, al);
                        be = fmaf(v, v, be);
                        ga = fmaf(u, v, ga);
                    }
#pragma unroll
                    for (int o = JG / 2; o > 0; o >>= 1) {
                        al += __shfl_xor_sync(gmask, al, o);
                        be += __shfl_xor_sync(gmask, be, o);
                        ga += __shfl_xor_sync(gmask, ga, o);
                    }
                    if (fabsf(ga) > JACOBI_TOL * sqrtf(al) * sqrtf(be)) {
                        const float zeta = (be - al) / (2.f * ga);
                        const float az = fabsf(zeta);
                        const float t = (az > 1e18f ? 0.5f / az : 1.f / (az + sqrtf(fmaf(az, az, 1.f))));
                        const float tt = zeta < 0.f ? -t : t;
                        // rotation [[c, s], [-s, c]] with c = 1/rr, s = t/rr applied as a
                        // correction: dc = 1 - c is formed directly, because for |t| < sqrt(eps)
                        // c rounds to 1 while s = t, and the rounded rotation would inflate column
                        // norms by t^2/2 each time (a systematic bias over thousands of rotations)
                        const float rr = sqrtf(fmaf(tt, tt, 1.f));
                        const float dc = (tt * tt) / (rr * (1.f + rr));
                        const float s = tt / rr;
                        for (int m = gl; m < n; m += JG) {
                            const float u = xa[m], v = xb[m];
                            xa[m] = u - fmaf(dc, u, s * v);
                            xb[m] = v - fmaf(dc, v, -s * u);
                        }
                        if (gl == 0 && t != 0.f) sFlag[0] = 1;
                    }
                }
                __syncthreads();
            }
            if (sFlag[0] == 0) {
                converged = true;
                break;
            }
            __syncthreads();
        }
        if (!converged && tid == 0) set_status(a.status, ISKV_ERR_NOT_CONVERGED);
        if (tid == 0 && a.stats) {
            atomicMax(a.stats, (unsigned long long)sweeps);
            atomicAdd(a.stats + 1, (unsigned long long)sweeps);
            atomicAdd(a.stats + 2, 1ull);
        }
    }

    // ---- singular values = column norms; select the top kp (descending, ties by index) -------
    for (int c = tid; c < N; c += FOLD_THREADS) {
        const float *x = c < k ? sC + c * LDS : sB + (c - k) * LDS;
        float s = 0.f;
        for (int m = 0; m < n; ++m) s = fmaf(x[m], x[m], s);
        s = sqrtf(s);
        if (!isfinite(s)) {
            set_status(a.status, ISKV_ERR_NONFINITE);
            s = -1.f;
        }
        sNrm[c] = s;
    }
    if (tid < 128) sSel[tid] = 0;
    __syncthreads();
    for (int c = tid; c < N; c += FOLD_THREADS) {
        const float s = sNrm[c];
        int rank = 0;
        for (int c2 = 0; c2 < N; ++c2) {
            const float s2 = sNrm[c2];
            rank += (s2 > s) || (s2 == s && c2 < c);
        }
        if (rank < kp) sSel[rank] = c;
    }
    __syncthreads();
    // normalise the selected columns in place: they become the columns of H (length n)
    for (int o = tid; o < kp * n; o += FOLD_THREADS) {
        const int c = o / n, m = o % n;
        const int cs = sSel[c];
        const float s = sNrm[cs];
        float *x = cs < k ? sC + cs * LDS : sB + (cs - k) * LDS;
        if (s > 1e-30f) x[m] = x[m] / s;
    }
    __syncthreads();
    // exactly-zero singular values: complete H with orthonormal directions (rare; rank-deficient
    // input); keeps B+ orthonormal
    if (warp == 0) {
        float *v = sScr;
        for (int c = 0; c < kp; ++c) {
            const int cs = sSel[c];
            if (sNrm[cs] > 1e-30f) continue;
            float *x = cs < k ? sC + cs * LDS : sB + (cs - k) * LDS;
            for (int e = 0; e < n; ++e) {
                for (int m = lane; m < n; m += 32) v[m] = (m == e) ? 1.f : 0.f;
                __syncwarp();
                for (int c2 = 0; c2 < kp; ++c2) {
                    const int cs2 = sSel[c2];
                    if (c2 == c || (sNrm[cs2] <= 1e-30f && c2 > c)) continue;
                    const float *y = cs2 < k ? sC + cs2 * LDS : sB + (cs2 - k) * LDS;
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
    for (int o = tid; o < D * k; o += FOLD_THREADS) {
        const int j = o / k, l = o % k;
        sA[(p + l) * LDS + j] = Bin[(size_t)j * r + l];
    }
    __syncthreads();
    // ---- sign convention: new basis vector c points along old basis vector c (H[c][c] >= 0) ----
    const int ks = k < kp ? k : kp;
    for (int c = tid; c < ks; c += FOLD_THREADS) {
        const int cs = sSel[c];
        const float *x = cs < k ? sC + cs * LDS : sB + (cs - k) * LDS;
        sTau[c] = x[c] < 0.f ? -1.f : 1.f;
    }
    __syncthreads();
    for (int o = tid; o < ks * n; o += FOLD_THREADS) {
        const int c = o / n, m = o % n;
        if (sTau[c] < 0.f) {
            const int cs = sSel[c];
            float *x = cs < k ? sC + cs * LDS : sB + (cs - k) * LDS;
            x[m] = -x[m];
        }
    }
    __syncthreads();

    // ---- outputs: Sigma+, H_top, B+ = [B P] H ------------------------------------------------
    float *sig_out = P.sigma + (size_t)unit * r;
    for (int c = tid; c < r; c += FOLD_THREADS) sig_out[c] = c < kp ? sNrm[sSel[c]] : 0.f;
    float *ht = P.htop + (size_t)unit * r * r;
    for (int o = tid; o < k * kp; o += FOLD_THREADS) {
        const int l = o / kp, c = o % kp;
        const int cs = sSel[c];
        const float *x = cs < k ? sC + cs * LDS : sB + (cs - k) * LDS;
        ht[(size_t)l * r + c] = x[l];
    }
    const int j = tid & (D - 1);
    const int c0 = tid >> 7;             // 0..3
    float bp[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int c = c0 + 4 * q;
        float s = 0.f;
        if (c < kp) {
            const int cs = sSel[c];
            const float *h = cs < k ? sC + cs * LDS : sB + (cs - k) * LDS;
            for (int l = 0; l < p; ++l) s = fmaf(sA[l * LDS + j], h[k + l], s);
            for (int l = 0; l < k; ++l) s = fmaf(sA[(p + l) * LDS + j], h[l], s);
        }
        bp[q] = s;
    }
    __syncthreads();                     // H and W consumed
    // ---- one Newton-Schulz step towards the nearest orthonormal basis, B+ <- B+ (3I - M) / 2 with
    //      M = B+^T B+ (the Jacobi stops at a relative orthogonality threshold, and without this
    //      the loss of orthonormality would add up over folds); H_top gets the same right factor so
    //      old coordinates stay consistent with the corrected basis.
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int c = c0 + 4 * q;
        if (c < kp) sC[c * LDS + j] = bp[q];
    }
    __syncthreads();
    for (int o = tid; o < kp * kp; o += FOLD_THREADS) {
        const int c = o / kp, c2 = o % kp;
        const float *x = sC + c * LDS, *y = sC + c2 * LDS;
        float s = 0.f;
        for (int jj = 0; jj < D; ++jj) s = fmaf(x[jj], y[jj], s);
        sB[o] = s;
    }
    for (int o = tid; o < k * kp; o += FOLD_THREADS) sA[o] = ht[(size_t)(o / kp) * r + o % kp];
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int c = c0 + 4 * q;
        if (c < kp) {
            float s = 0.f;
            for (int c2 = 0; c2 < kp; ++c2) s = fmaf(sC[c2 * LDS + j], sB[c2 * kp + c], s);
            bp[q] = 1.5f * bp[q] - 0.5f * s;
        }
    }
    for (int o = tid; o < k * kp; o += FOLD_THREADS) {
        const int l = o / kp, c = o % kp;
        float s = 0.f;
        for (int c2 = 0; c2 < kp; ++c2) s = fmaf(sA[l * kp + c2], sB[c2 * kp + c], s);
        ht[(size_t)l * r + c] = 1.5f * sA[o] - 0.5f * s;
    }
    float *Bout = P.basis_out + (size_t)unit * D * r;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int c = c0 + 4 * q;
        if (c < r) Bout[(size_t)j * r + c] = bp[q];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int c = c0 + 4 * q;
        if (c < kp) sC[c * LDS + j] = bp[q];
    }
    // reload F for the new rows' coordinates
    for (int o = tid; o < b * D; o += FOLD_THREADS) {
        const int i = o / D, jj = o % D;
        const int slot = (a.slot0 + i) % a.R;
        sA[i * LDS + jj] = load_row_elem(P.ring, ring_base + (size_t)slot * D + jj, a.kv_dtype);
    }
    __syncthreads();
    // ---- new rows' coordinates C[n_c + i] = F[i] B+ --------------------------------------------
    float *Cn = P.coords + ((size_t)unit * a.n_max + a.n_c) * r;
    for (int o = tid; o < b * r; o += FOLD_THREADS) {
        const int i = o / r, c = o % r;
        float s = 0.f;
        if (c < kp) {
            const float *f = sA + i * LDS, *bc = sC + c * LDS;
            for (int jj = 0; jj < D; ++jj) s = fmaf(f[jj], bc[jj], s);
        }
        Cn[(size_t)i * r + c] = s;
    }
}

// History rotation: old coordinates move with the basis, C[0:n] <- C[0:n] H[:k] (iS-KV summary,
// "Block-Incremental Decoding Updates", U+ = diag(U, I_b) G, so the old rows of U+ Sigma+ are
// U Sigma H[:k]). Stale mode keeps the old coordinates (zero-padded to the new rank).
constexpr int ROT_ROWS = 64;
constexpr int ROT_THREADS = 256;

__global__ void __launch_bounds__(ROT_THREADS) rotate_kernel(RotArgs a) {
    extern __shared__ float smem[];
    const RotPath P = blockIdx.z ? a.path[1] : a.path[0];
    const int unit = a.unit0 + blockIdx.y;
    const long long row0 = (long long)blockIdx.x * ROT_ROWS;
    if (row0 >= a.n_old) return;
    const int rows = (int)min((long long)ROT_ROWS, a.n_old - row0);
    const int k = P.k, kp = P.kp, r = P.r;
    float *sH = smem;                         // k x kp
    float *sX = sH + r * r;                   // ROT_ROWS x (k + 1)
    float *C = P.coords + ((size_t)unit * a.n_max + row0) * r;
    if (!a.stale) {
        const float *ht = P.htop + (size_t)unit * r * r;
        for (int o = threadIdx.x; o < k * kp; o += ROT_THREADS) {
            const int l = o / kp, c = o % kp;
            sH[l * kp + c] = ht[(size_t)l * r + c];
        }
    }
    for (int o = threadIdx.x; o < rows * k; o += ROT_THREADS) {
        const int i = o / k, l = o % k;
        sX[i * (k + 1) + l] = C[(size_t)i * r + l];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < rows * r; o += ROT_THREADS) {
        const int i = o / r, c = o % r;
        float s = 0.f;
        if (a.stale) {
            s = c < k ? sX[i * (k + 1) + c] : 0.f;
        } else if (c < kp) {
            const float *x = sX + i * (k + 1);
            for (int l = 0; l < k; ++l) s = fmaf(x[l], sH[l * kp + c], s);
        }
        C[(size_t)i * r + c] = s;
    }
}

cudaError_t launch_fold(const FoldArgs &a, int n_units, cudaStream_t s) {
    static bool attr_set = false;
    const size_t smem = fold_smem_bytes();
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(fold_core_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    fold_core_kernel<<<dim3(n_units, 2), FOLD_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_rotate(const RotArgs &a, int n_units, cudaStream_t s) {
    if (a.n_old <= 0) return cudaSuccess;
    const int rmax = a.path[0].r > a.path[1].r ? a.path[0].r : a.path[1].r;
    const size_t smem = (size_t)(rmax * rmax + ROT_ROWS * (rmax + 1)) * sizeof(float);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(rotate_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)((128 * 128 + ROT_ROWS * 129) * sizeof(float)));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const unsigned gx = (unsigned)((a.n_old + ROT_ROWS - 1) / ROT_ROWS);
    rotate_kernel<<<dim3(gx, n_units, 2), ROT_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace iskv
