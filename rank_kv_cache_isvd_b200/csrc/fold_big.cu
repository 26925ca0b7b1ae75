// Folds of blocks larger than the in-shared-memory fold kernel holds (b > 128 rows).
//
// iS-KV summary, "Block-Incremental Decoding Updates": the fold needs the core
// Z = [[Sigma, 0], [F B, F P]] only through its singular values and right singular vectors
// (Sigma+, H; the new basis is [B P] H and old coordinates move by H[:k]). Both depend on F only
// through F^T F, so any 128-row F~ with F~^T F~ = F^T F gives the same Sigma+, H and basis: F~ is
// the triangular factor R of a QR of F. The fold of a large block is therefore
//   1. rfactor_kernel: R of the b x 128 block, by Householder QR of [R; next 128 rows] over the
//      block's 128-row chunks (tall-skinny QR), written as a 128-row fp32 pseudo-block;
//   2. the regular fold kernel on that pseudo-block (its new-row coordinates are skipped);
//   3. newrows_kernel: coordinates of the block's real rows, C[n_c + i] = F[i] B+.
// With b > 128 >= d - k the residual basis P is the complement of B in both forms.
#include "iskv_internal.cuh"

namespace iskv {

constexpr int RF_THREADS = 256;
constexpr int RF_LDM = 2 * DEC_TILE + 1;      // column stride of the stacked [R; chunk] matrix

__device__ __forceinline__ float rf_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA per (unit, path): R (128 x 128, upper triangular, row i in pseudo-block row i) of the
// block F = ring rows slot0 .. slot0 + b - 1 (mod R_ring).
__global__ void __launch_bounds__(RF_THREADS) rfactor_kernel(RFactorArgs a) {
    extern __shared__ float rsm[];
    float *M = rsm;                              // [128 columns][RF_LDM]: rows 0..127 = R, 128.. = chunk
    float *sTau = rsm + D * RF_LDM;
    const RFactorPath P = (a.path_lo + (int)blockIdx.y) ? a.path[1] : a.path[0];
    const int unit = a.unit0 + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int FW = RF_THREADS / 32;
    for (int o = tid; o < D * RF_LDM; o += RF_THREADS) M[o] = 0.f;
    __syncthreads();
    const size_t ring_base = (size_t)unit * a.R * D;
    for (int c0 = 0; c0 < a.b; c0 += DEC_TILE) {
        const int rows = min(DEC_TILE, a.b - c0);
        // chunk rows into M rows 128 .. 128 + rows - 1 (zero below)
        for (int o = tid; o < DEC_TILE * D; o += RF_THREADS) {
            const int i = o / D, j = o % D;
            float v = 0.f;
            if (i < rows) {
                if (P.src != nullptr) {
                    // prefill: the caller's rows; protected rows do not enter the factor
                    const long long p = c0 + i;
                    if (!(P.fbit && (a.flags[(size_t)unit * a.flag_stride + p] & P.fbit)))
                        v = load_row_elem(P.src, ((size_t)blockIdx.x * a.src_rows + p) * D + j, a.kv_dtype);
                } else {
                    const int slot = (a.slot0 + c0 + i) % a.R;
                    v = load_row_elem(P.ring, ring_base + (size_t)slot * D + j, a.kv_dtype);
                }
            }
            M[j * RF_LDM + DEC_TILE + i] = v;
        }
        __syncthreads();
        // Householder QR of the 256 x 128 matrix M (columns jc = 0 .. 127)
        const int m = 2 * DEC_TILE;
        for (int jc = 0; jc < D; ++jc) {
            float *col = M + jc * RF_LDM;
            if (warp == 0) {
                float xv[8], s2 = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = lane + 32 * u;
                    xv[u] = col[i];
                    s2 = fmaf(i > jc ? xv[u] : 0.f, xv[u], s2);
                }
                s2 = rf_warp_sum(s2);
                const float alpha = col[jc];
                float tau = 0.f, beta = alpha, scale = 0.f;
                if (s2 > 0.f) {
                    beta = -copysignf(sqrtf(fmaf(alpha, alpha, s2)), alpha);
                    tau = (beta - alpha) / beta;
                    scale = 1.f / (alpha - beta);
                }
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = lane + 32 * u;
                    if (i > jc) col[i] = xv[u] * scale;
                }
                if (lane == 0) {
                    col[jc] = beta;
                    sTau[jc] = tau;
                }
            }
            __syncthreads();
            const float tau = sTau[jc];
            if (tau != 0.f) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = lane + 32 * u;
                    v[u] = i > jc ? col[i] : 0.f;
                }
                for (int c = jc + 1 + warp; c < D; c += FW) {
                    float *x = M + c * RF_LDM;
                    float w = 0.f, xq[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        xq[u] = x[lane + 32 * u];
                        w = fmaf(v[u], xq[u], w);
                    }
                    w = rf_warp_sum(w);
                    const float xj = x[jc];
                    __syncwarp();
                    const float wq = (w + xj) * tau;
                    if (lane == 0) x[jc] = xj - wq;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int i = lane + 32 * u;
                        if (i > jc) x[i] = fmaf(-wq, v[u], xq[u]);
                    }
                    __syncwarp();
                }
            }
            __syncthreads();
        }
        // keep R (upper triangle of rows 0..127); clear the reflectors below it
        for (int o = tid; o < D * m; o += RF_THREADS) {
            const int jc = o / m, i = o % m;
            if (i > jc) M[jc * RF_LDM + i] = 0.f;
        }
        __syncthreads();
    }
    // pseudo-block row i = R[i][:] (fp32)
    float *out = P.rout + (size_t)unit * DEC_TILE * D;
    for (int o = tid; o < DEC_TILE * D; o += RF_THREADS) {
        const int i = o / D, j = o % D;
        out[(size_t)i * D + j] = M[j * RF_LDM + i];
    }
}

// One CTA per (128-row chunk, unit, path): C[n_c + i] = F[i] B+ for the block's real rows.
__global__ void __launch_bounds__(RF_THREADS) newrows_kernel(NewRowsArgs a) {
    extern __shared__ float nsm[];
    const NewRowsPath P = (a.path_lo + (int)blockIdx.z) ? a.path[1] : a.path[0];
    const int unit = a.unit0 + blockIdx.y;
    const int r = P.r, kp = P.kp, ldb = kp | 1;
    float *sB = nsm;                                 // B+ [D][ldb]
    float *sF = nsm + D * ldb;                       // F rows [32][D + 1]
    const float *Bp = P.basis + (size_t)unit * D * r;
    for (int o = threadIdx.x; o < D * kp; o += RF_THREADS)
        sB[(o / kp) * ldb + o % kp] = Bp[(size_t)(o / kp) * r + o % kp];
    const size_t ring_base = (size_t)unit * a.R * D;
    const int c0 = blockIdx.x * DEC_TILE;
    const int rows = min(DEC_TILE, a.b - c0);
    for (int s0 = 0; s0 < rows; s0 += 32) {
        __syncthreads();
        const int sr = min(32, rows - s0);
        for (int o = threadIdx.x; o < 32 * D; o += RF_THREADS) {
            const int i = o / D, j = o % D;
            float v = 0.f;
            if (i < sr) {
                if (P.src != nullptr) {
                    // prefill: the caller's rows; protected rows get zero coordinates
                    const long long p = c0 + s0 + i;
                    if (!(P.fbit && (a.flags[(size_t)unit * a.flag_stride + p] & P.fbit)))
                        v = load_row_elem(P.src, ((size_t)blockIdx.y * a.src_rows + p) * D + j, a.kv_dtype);
                } else {
                    const int slot = (a.slot0 + c0 + s0 + i) % a.R;
                    v = load_row_elem(P.ring, ring_base + (size_t)slot * D + j, a.kv_dtype);
                }
            }
            sF[i * (D + 1) + j] = v;
        }
        __syncthreads();
        for (int o = threadIdx.x; o < sr * r; o += RF_THREADS) {
            const int i = o / r, c = o % r;
            float s = 0.f;
            if (c < kp) {
                const float *f = sF + i * (D + 1);
                for (int j = 0; j < D; ++j) s = fmaf(f[j], sB[j * ldb + c], s);
            }
            store_coord(P.coords, ((size_t)unit * a.n_max + a.n_c + c0 + s0 + i) * r + c, s, a.cbf);
        }
    }
}

size_t rfactor_smem_bytes() { return ((size_t)D * RF_LDM + D) * sizeof(float); }

cudaError_t launch_rfactor(const RFactorArgs &a, int n_units, cudaStream_t s) {
    if (a.path_hi <= a.path_lo || n_units <= 0) return cudaSuccess;
    static size_t attr[64] = {0};
    const cudaError_t e = ensure_smem((const void *)rfactor_kernel, rfactor_smem_bytes(), attr);
    if (e != cudaSuccess) return e;
    rfactor_kernel<<<dim3(n_units, a.path_hi - a.path_lo), RF_THREADS, rfactor_smem_bytes(), s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_newrows(const NewRowsArgs &a, int n_units, cudaStream_t s) {
    if (a.path_hi <= a.path_lo || n_units <= 0) return cudaSuccess;
    const int kpmax = a.path[0].kp > a.path[1].kp ? a.path[0].kp : a.path[1].kp;
    const size_t smem = ((size_t)D * (kpmax | 1) + 32 * (D + 1)) * sizeof(float);
    static size_t attr[64] = {0};
    const cudaError_t e = ensure_smem((const void *)newrows_kernel, smem, attr);
    if (e != cudaSuccess) return e;
    const int chunks = (a.b + DEC_TILE - 1) / DEC_TILE;
    newrows_kernel<<<dim3(chunks, n_units, a.path_hi - a.path_lo), RF_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace iskv
