// Prefill with key/value protection.
//
// iS-KV summary, "Prefill Compression":
//   1. key protection: the prefill's keys are cut into chunks of consecutive positions; chunk c of
//      kv-head h scores s_{c,h} = min_{i in c} cos(k_i^rot, mean_c k^rot) (keys rotated at their
//      positions); the m lowest-scoring chunks, plus a local suffix, are the protected key
//      positions P_K;
//   2. value protection: P_V holds every position within rho tokens of P_K;
//   3. the remaining rows are factorised by a truncated SVD.
// Protected rows stay exact ("Reconstruction and Storage": X~[i] is the exact row for i in E_X).
//
// prot_score_kernel: one CTA per (chunk, unit) computes the chunk's score in fp32.
// prot_select_kernel: one CTA per unit picks the m lowest scores (ties by chunk index), marks
//   P_K (bit 0) and P_V (bit 1) in a per-position flag byte, and copies the protected rows with
//   their positions, in position order, into the unit's protected store.
// The truncated SVD of the remaining rows reuses the large-block fold: the triangular factor of
// the rows (flagged rows read as zero, so they do not enter it), the fold of that factor from
// rank 0, and the coordinates X[i] B+ of every row (zero for flagged rows).
#include <math_constants.h>

#include "iskv_internal.cuh"

namespace iskv {

constexpr int PS_THREADS = 128;
constexpr int SEL_THREADS = 256;

__device__ __forceinline__ float ps_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA per (chunk, unit): rows [c chunk, min(end, (c + 1) chunk)) of the unit's keys.
__global__ void __launch_bounds__(PS_THREADS) prot_score_kernel(ProtArgs a) {
    extern __shared__ float psm[];                 // [chunk][D + 1] rotated keys, then [D] mean
    const int c = blockIdx.x;
    const int ul = blockIdx.y;                     // unit within the call's units
    const long long r0 = (long long)c * a.chunk;
    const int rows = (int)min((long long)a.chunk, a.end - r0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *sK = psm;
    float *sM = psm + a.chunk * (D + 1);
    float *sRed = sM + D;                          // [4]
    const size_t base = (size_t)ul * a.src_rows;
    // rotate pair j of every row (threads 0 .. 63), position = row index
    for (int o = tid; o < rows * DH; o += PS_THREADS) {
        const int i = o / DH, j = o % DH;
        const long long pos = r0 + i;
        const float x = load_row_elem(a.keys, (base + pos) * D + j, a.kv_dtype);
        const float y = load_row_elem(a.keys, (base + pos) * D + DH + j, a.kv_dtype);
        float cs = 1.f, sn = 0.f;
        if (a.rope_cs != nullptr) {
            const float2 t = a.rope_cs[(size_t)pos * DH + j];
            cs = t.x;
            sn = t.y;
        }
        sK[i * (D + 1) + j] = fmaf(x, cs, -y * sn);
        sK[i * (D + 1) + DH + j] = fmaf(y, cs, x * sn);
    }
    __syncthreads();
    {
        float s = 0.f;
        for (int i = 0; i < rows; ++i) s += sK[i * (D + 1) + tid];
        sM[tid] = s / (float)rows;
    }
    __syncthreads();
    float mm = sM[tid] * sM[tid];
    mm = ps_warp_sum(mm);
    if (lane == 0) sRed[warp] = mm;
    __syncthreads();
    const float nm = sqrtf((sRed[0] + sRed[1]) + (sRed[2] + sRed[3]));
    // each warp takes rows warp, warp + 4, ...: cosine with the mean, min over the chunk
    float mn = CUDART_INF_F;
    for (int i = warp; i < rows; i += 4) {
        float dt = 0.f, nn = 0.f;
        for (int j = lane; j < D; j += 32) {
            const float v = sK[i * (D + 1) + j];
            dt = fmaf(v, sM[j], dt);
            nn = fmaf(v, v, nn);
        }
        dt = ps_warp_sum(dt);
        nn = ps_warp_sum(nn);
        const float nr = sqrtf(nn);
        const float cs = (nr > 0.f && nm > 0.f) ? dt / (nr * nm) : 1.f;
        mn = fminf(mn, cs);
    }
    __syncthreads();
    if (lane == 0) sRed[warp] = mn;
    __syncthreads();
    if (tid == 0)
        a.scores[(size_t)ul * a.n_chunks_cap + c] =
            fminf(fminf(sRed[0], sRed[1]), fminf(sRed[2], sRed[3]));
}

// One CTA per unit: outlier chunks, flags, and the protected stores.
__global__ void __launch_bounds__(SEL_THREADS) prot_select_kernel(ProtArgs a) {
    extern __shared__ float ssm[];
    float *sc = ssm;                                           // [n_chunks] scores
    float *rv = sc + a.n_chunks;                               // [SEL_THREADS] reduction values
    int *ri = reinterpret_cast<int *>(rv + SEL_THREADS);       // [SEL_THREADS] reduction indices
    int *sel = ri + SEL_THREADS;                               // [m] selected chunks
    int *cnt = sel + (a.m > 0 ? a.m : 1);                      // [SEL_THREADS + 1] scan
    const int ul = blockIdx.x;
    const int unit = a.unit0 + ul;
    const int tid = threadIdx.x;
    for (int c = tid; c < a.n_chunks; c += SEL_THREADS) sc[c] = a.scores[(size_t)ul * a.n_chunks_cap + c];
    __syncthreads();
    const int msel = a.m < a.n_chunks ? a.m : a.n_chunks;
    int *nsel_s = cnt + SEL_THREADS + 1;
    if (tid == 0) *nsel_s = 0;
    for (int r = 0; r < msel; ++r) {
        __syncthreads();                         // the previous round's reads are done
        float best = CUDART_INF_F;
        int bi = 0x7fffffff;
        for (int c = tid; c < a.n_chunks; c += SEL_THREADS) {
            const float v = sc[c];               // taken chunks hold +inf; NaN never compares less
            if (v < best || (v == best && v != CUDART_INF_F && c < bi)) {
                best = v;
                bi = c;
            }
        }
        rv[tid] = best;
        ri[tid] = bi;
        __syncthreads();
        for (int o = SEL_THREADS / 2; o > 0; o >>= 1) {
            if (tid < o) {
                const float v = rv[tid + o];
                const int i = ri[tid + o];
                if (v < rv[tid] || (v == rv[tid] && i < ri[tid])) {
                    rv[tid] = v;
                    ri[tid] = i;
                }
            }
            __syncthreads();
        }
        if (tid == 0 && ri[0] >= 0 && ri[0] < a.n_chunks) {
            sel[(*nsel_s)++] = ri[0];
            sc[ri[0]] = CUDART_INF_F;
        }
    }
    __syncthreads();
    const int nsel = *nsel_s;
    // P_K: selected chunks and the suffix
    unsigned char *fl = a.flags + (size_t)unit * a.flag_stride;
    for (long long p = tid; p < a.end; p += SEL_THREADS) {
        bool k = p >= a.end - a.suffix;            // the positions just before the window
        const int c = (int)(p / a.chunk);
        for (int r = 0; r < nsel && !k; ++r) k = sel[r] == c;
        fl[p] = k ? 1 : 0;
    }
    __syncthreads();
    // P_V: within rho of P_K
    for (long long p = tid; p < a.end; p += SEL_THREADS) {
        bool v = false;
        const long long lo = p - a.rho > 0 ? p - a.rho : 0;
        const long long hi = p + a.rho < a.end - 1 ? p + a.rho : a.end - 1;
        for (long long q = lo; q <= hi && !v; ++q) v = (fl[q] & 1) != 0;
        if (v) fl[p] |= 2;
    }
    __syncthreads();
    // protected stores, in position order: a block scan of the per-thread counts over contiguous
    // position ranges
    const long long per = (a.end + SEL_THREADS - 1) / SEL_THREADS;
    const long long p0 = tid * per, p1 = p0 + per < a.end ? p0 + per : a.end;
    for (int x = 0; x < 2; ++x) {
        const unsigned char bit = (unsigned char)(1u << x);
        int my = 0;
        for (long long p = p0; p < p1; ++p) my += (fl[p] & bit) ? 1 : 0;
        cnt[tid] = my;
        __syncthreads();
        if (tid == 0) {
            int run = 0;
            for (int t = 0; t < SEL_THREADS; ++t) {
                const int v = cnt[t];
                cnt[t] = run;
                run += v;
            }
            cnt[SEL_THREADS] = run;
        }
        __syncthreads();
        int at = cnt[tid];
        const size_t esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
        for (long long p = p0; p < p1; ++p) {
            if (!(fl[p] & bit)) continue;
            if (at < a.cap) {
                a.ppos[x][(size_t)unit * a.cap + at] = (int)p;
                const char *src = static_cast<const char *>(a.src[x]) + ((size_t)ul * a.src_rows + p) * D * esz;
                char *dst = static_cast<char *>(a.store[x]) + ((size_t)unit * a.cap + at) * D * esz;
                for (size_t b = 0; b < D * esz; b += 16)
                    *reinterpret_cast<uint4 *>(dst + b) = *reinterpret_cast<const uint4 *>(src + b);
            }
            ++at;
        }
        __syncthreads();
        if (tid == 0) {
            const int total = cnt[SEL_THREADS];
            a.pcount[x][unit] = total < a.cap ? total : a.cap;
            if (total > a.cap) set_status(a.status, ISKV_ERR_CAPACITY);
        }
        __syncthreads();
    }
}

size_t prot_score_smem(int chunk) { return ((size_t)chunk * (D + 1) + D + 4) * sizeof(float); }
size_t prot_select_smem(int n_chunks, int m) {
    return ((size_t)n_chunks + SEL_THREADS) * sizeof(float) +
           ((size_t)SEL_THREADS + (m > 0 ? m : 1) + SEL_THREADS + 2) * sizeof(int);
}

cudaError_t launch_protect(const ProtArgs &a, int n_units, cudaStream_t s) {
    static size_t attr_s[64] = {0}, attr_p[64] = {0};
    const size_t s1 = prot_score_smem(a.chunk), s2 = prot_select_smem(a.n_chunks, a.m);
    cudaError_t e = ensure_smem((const void *)prot_score_kernel, s1, attr_s);
    if (e != cudaSuccess) return e;
    e = ensure_smem((const void *)prot_select_kernel, s2, attr_p);
    if (e != cudaSuccess) return e;
    prot_score_kernel<<<dim3(a.n_chunks, n_units), PS_THREADS, s1, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prot_select_kernel<<<n_units, SEL_THREADS, s2, s>>>(a);
    return cudaGetLastError();
}

}  // namespace iskv
