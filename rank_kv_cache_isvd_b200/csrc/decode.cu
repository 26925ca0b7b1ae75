// Decode attention over the compressed history plus the exact window.
//
// iS-KV summary, "Reconstruction and Storage": compressed key/value rows are (C B^T)[i] and the
// window rows are exact. Keys were compressed before RoPE, so each reconstructed key is rotated at
// its own position before the dot product with the (already rotated) query. Values never leave
// rank space inside a split: each split accumulates sum_i p_i C_V[i] (r_V numbers per q-head),
// and the combine kernel expands the log-sum-exp-merged sum once through B_V^T.
//
// decode_split_kernel: grid (splits, units of the layer); a split covers up to split_rows
// compressed positions or one 128-row tile of the window; each CTA serves the G q-heads of its
// kv-head and writes (max, sum, accumulator) partials. decode_combine_kernel merges them.
#include <math_constants.h>

#include "iskv_internal.cuh"

namespace iskv {

constexpr int DEC_THREADS = 256;

struct DecSmem {
    // offsets in floats
    int bt, q, ck, cv, s, stat;
    int total;
};

__host__ __device__ inline DecSmem dec_layout(int rK, int G) {
    DecSmem L;
    const int ldk = rK | 1;
    L.bt = 0;                                 // B_K^T: [rK][D]
    L.q = L.bt + rK * D;                      // q: [G][D] (pre-scaled)
    L.ck = L.q + GMAX * D;                    // C_K tile: [128][ldk]
    L.cv = L.ck + DEC_TILE * ldk;             // C_V tile [128][rV] or V rows [128][D]
    L.s = L.cv + DEC_TILE * D;                // scores/probabilities [G][128]
    L.stat = L.s + GMAX * DEC_TILE;           // m[G], l[G], alpha[G]
    L.total = L.stat + 3 * GMAX;
    (void)G;
    return L;
}

__global__ void __launch_bounds__(DEC_THREADS) decode_split_kernel(DecodeArgs a) {
    extern __shared__ float smem[];
    const int rK = a.r[0], rV = a.r[1], kK = a.k[0], kV = a.k[1];
    const DecSmem L = dec_layout(rK, a.G);
    float *sBt = smem + L.bt, *sQ = smem + L.q, *sCk = smem + L.ck, *sCv = smem + L.cv;
    float *sS = smem + L.s, *sM = smem + L.stat, *sL = sM + GMAX, *sAl = sL + GMAX;
    const int ldk = rK | 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = a.G;
    const int ul = blockIdx.y;                 // unit within the layer: s * H + h
    const int split = blockIdx.x;
    const int seq = ul / a.H, h = ul % a.H;
    const bool comp = split < a.n_split_c;
    long long p0, p1;
    if (comp) {
        p0 = (long long)split * a.split_rows;
        p1 = min(a.n_c, p0 + a.split_rows);
    } else {
        p0 = a.n_c + (long long)(split - a.n_split_c) * DEC_TILE;
        p1 = min(a.t, p0 + DEC_TILE);
    }
    // q (pre-scaled by 1/sqrt(d)) and the key basis
    for (int o = tid; o < G * D; o += DEC_THREADS)
        sQ[o] = a.q[((size_t)seq * a.H * G + (size_t)h * G) * D + o] * a.scale;
    if (comp)
        for (int o = tid; o < D * kK; o += DEC_THREADS) {
            const int j = o / kK, c = o % kK;
            sBt[c * D + j] = a.basis[0][((size_t)ul * D + j) * rK + c];
        }
    if (tid < G) {
        sM[tid] = -CUDART_INF_F;
        sL[tid] = 0.f;
    }
    const int nacc = comp ? kV : D;            // accumulator width per q-head
    float vacc[4] = {0.f, 0.f, 0.f, 0.f};

    const int q4 = tid & 3, rp = tid >> 2;     // channel quarter, row pair
    const long long cu = coord_unit(ul, a.cdiv);     // the kv-head's coordinate unit
    const float *Ck = static_cast<const float *>(a.coords[0]) + (size_t)cu * a.n_max * rK;
    const float *Cv = static_cast<const float *>(a.coords[1]) + (size_t)cu * a.n_max * rV;
    const size_t ring_base = (size_t)ul * a.R * D;

    for (long long t0 = p0; t0 < p1; t0 += DEC_TILE) {
        const int rows = (int)min((long long)DEC_TILE, p1 - t0);
        __syncthreads();
        // ---- stage the tile ------------------------------------------------------------------
        if (comp) {
            for (int o = tid; o < DEC_TILE * kK; o += DEC_THREADS) {
                const int i = o / kK, c = o % kK;
                sCk[i * ldk + c] = i < rows ? Ck[(size_t)(t0 + i) * rK + c] : 0.f;
            }
            for (int o = tid; o < DEC_TILE * kV; o += DEC_THREADS) {
                const int i = o / kV, c = o % kV;
                sCv[i * kV + c] = i < rows ? Cv[(size_t)(t0 + i) * rV + c] : 0.f;
            }
        } else {
            for (int o = tid; o < DEC_TILE * D; o += DEC_THREADS) {
                const int i = o / D, j = o % D;
                float v = 0.f;
                if (i < rows) {
                    const int slot = (int)((t0 + i) % a.R);
                    v = load_row_elem(a.ring[1], ring_base + (size_t)slot * D + j, a.kv_dtype);
                }
                sCv[o] = v;
            }
        }
        __syncthreads();
        // ---- keys for rows 2rp, 2rp+1, channels lo = 16u + 4q4 + v, hi = lo + 64 ------------
        float kx[2][32];
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int q = 0; q < 32; ++q) kx[e][q] = 0.f;
        if (comp) {
            const float *c0p = sCk + (2 * rp) * ldk, *c1p = c0p + ldk;
            for (int c = 0; c < kK; ++c) {
                const float c0 = c0p[c], c1 = c1p[c];
                const float *bt = sBt + c * D + 4 * q4;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 lo = *reinterpret_cast<const float4 *>(bt + 16 * u);
                    const float4 hi = *reinterpret_cast<const float4 *>(bt + 64 + 16 * u);
                    const float l4[4] = {lo.x, lo.y, lo.z, lo.w}, h4[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        kx[0][8 * u + v] = fmaf(c0, l4[v], kx[0][8 * u + v]);
                        kx[0][8 * u + 4 + v] = fmaf(c0, h4[v], kx[0][8 * u + 4 + v]);
                        kx[1][8 * u + v] = fmaf(c1, l4[v], kx[1][8 * u + v]);
                        kx[1][8 * u + 4 + v] = fmaf(c1, h4[v], kx[1][8 * u + 4 + v]);
                    }
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = 2 * rp + e;
                if (i < rows) {
                    const int slot = (int)((t0 + i) % a.R);
                    const size_t base = ring_base + (size_t)slot * D;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int j = 16 * u + 4 * q4 + v;
                            kx[e][8 * u + v] = load_row_elem(a.ring[0], base + j, a.kv_dtype);
                            kx[e][8 * u + 4 + v] = load_row_elem(a.ring[0], base + j + DH, a.kv_dtype);
                        }
                }
            }
        }
        // ---- RoPE at the row's position, then partial scores for the G q-heads ---------------
        float part[2][GMAX];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const long long pos = t0 + 2 * rp + e;
            const bool valid = (2 * rp + e) < rows;
#pragma unroll
            for (int g = 0; g < GMAX; ++g) part[e][g] = 0.f;
            if (valid && a.rope_cs) {
                const float2 *cs = a.rope_cs + pos * DH;
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float2 w = cs[16 * u + 4 * q4 + v];
                        const float xl = kx[e][8 * u + v], xh = kx[e][8 * u + 4 + v];
                        kx[e][8 * u + v] = xl * w.x - xh * w.y;
                        kx[e][8 * u + 4 + v] = xh * w.x + xl * w.y;
                    }
            }
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                if (g < G) {
                    const float *qg = sQ + g * D + 4 * q4;
                    float s = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 ql = *reinterpret_cast<const float4 *>(qg + 16 * u);
                        const float4 qh = *reinterpret_cast<const float4 *>(qg + 64 + 16 * u);
                        s = fmaf(ql.x, kx[e][8 * u + 0], s);
                        s = fmaf(ql.y, kx[e][8 * u + 1], s);
                        s = fmaf(ql.z, kx[e][8 * u + 2], s);
                        s = fmaf(ql.w, kx[e][8 * u + 3], s);
                        s = fmaf(qh.x, kx[e][8 * u + 4], s);
                        s = fmaf(qh.y, kx[e][8 * u + 5], s);
                        s = fmaf(qh.z, kx[e][8 * u + 6], s);
                        s = fmaf(qh.w, kx[e][8 * u + 7], s);
                    }
                    part[e][g] = s;
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                float s = part[e][g];
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                part[e][g] = s;
            }
        if (q4 == 0) {
#pragma unroll
            for (int g = 0; g < GMAX; ++g)
                if (g < G) {
                    sS[g * DEC_TILE + 2 * rp] = part[0][g];
                    sS[g * DEC_TILE + 2 * rp + 1] = part[1][g];
                }
        }
        __syncthreads();
        // ---- online softmax (warp g handles q-head g) -----------------------------------------
        if (warp < G) {
            const int g = warp;
            float sv[4], mt = -CUDART_INF_F;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = lane + 32 * q;
                sv[q] = i < rows ? sS[g * DEC_TILE + i] : -CUDART_INF_F;
                mt = fmaxf(mt, sv[q]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
            const float m_old = sM[g];
            const float m_new = fmaxf(m_old, mt);
            const float alpha = expf(m_old - m_new);
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = lane + 32 * q;
                const float pr = i < rows ? expf(sv[q] - m_new) : 0.f;
                sS[g * DEC_TILE + i] = pr;
                sum += pr;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            __syncwarp();
            if (lane == 0) {
                sL[g] = sL[g] * alpha + sum;
                sM[g] = m_new;
                sAl[g] = alpha;
            }
        }
        __syncthreads();
        // ---- value accumulation: acc[g][c] = acc * alpha_g + sum_i p[g][i] V[i][c] --------------
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int o = tid + DEC_THREADS * w;
            if (o < G * nacc) {
                const int g = o / nacc, c = o % nacc;
                const float *pg = sS + g * DEC_TILE;
                float s = vacc[w] * sAl[g];
                for (int i = 0; i < rows; ++i) s = fmaf(pg[i], sCv[i * nacc + c], s);
                vacc[w] = s;
            }
        }
    }
    __syncthreads();
    // ---- partials: [m, l, acc[nacc]] per q-head ---------------------------------------------
    float *ws = a.ws + ((size_t)ul * a.max_splits + split) * G * (2 + D);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int o = tid + DEC_THREADS * w;
        if (o < G * nacc) {
            const int g = o / nacc, c = o % nacc;
            ws[g * (2 + D) + 2 + c] = vacc[w];
        }
    }
    if (tid < G) {
        ws[tid * (2 + D)] = sM[tid];
        ws[tid * (2 + D) + 1] = sL[tid];
    }
}

// One CTA per unit of the layer, 128 threads: log-sum-exp merge of the splits, rank-space value
// sum expanded once through B_V^T, plus the window splits' exact-value sums.
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeArgs a) {
    __shared__ float sAcc[D];
    const int ul = blockIdx.x;
    const int seq = ul / a.H, h = ul % a.H;
    const int j = threadIdx.x;
    const int G = a.G, rV = a.r[1], kV = a.k[1];
    const float *ws = a.ws + (size_t)ul * a.max_splits * G * (2 + D);
    const float *BV = a.basis[1] + (size_t)ul * D * rV;
    for (int g = 0; g < G; ++g) {
        float M = -CUDART_INF_F;
        for (int s = 0; s < a.n_split; ++s) M = fmaxf(M, ws[((size_t)s * G + g) * (2 + D)]);
        float Lsum = 0.f, acc_w = 0.f, acc_r = 0.f;
        for (int s = 0; s < a.n_split; ++s) {
            const float *pw = ws + ((size_t)s * G + g) * (2 + D);
            const float w = expf(pw[0] - M);
            Lsum = fmaf(w, pw[1], Lsum);
            if (s < a.n_split_c) {
                if (j < kV) acc_r = fmaf(w, pw[2 + j], acc_r);
            } else {
                acc_w = fmaf(w, pw[2 + j], acc_w);
            }
        }
        __syncthreads();
        sAcc[j] = acc_r;
        __syncthreads();
        float o = acc_w;
        for (int c = 0; c < kV; ++c) o = fmaf(sAcc[c], BV[(size_t)j * rV + c], o);
        a.out[((size_t)seq * a.H * G + (size_t)h * G + g) * D + j] = o / Lsum;
    }
}

cudaError_t launch_decode(const DecodeArgs &a, int n_units, cudaStream_t s) {
    const DecSmem L = dec_layout(a.r[0], a.G);
    const size_t smem = (size_t)L.total * sizeof(float);
    static size_t attr[64] = {0};
    cudaError_t e = ensure_smem((const void *)decode_split_kernel, smem, attr);
    if (e != cudaSuccess) return e;
    decode_split_kernel<<<dim3(a.n_split, n_units), DEC_THREADS, smem, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<<<n_units, D, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace iskv
