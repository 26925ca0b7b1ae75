// Exact recent window (ring buffer of window + block rows per unit and path), cache
// reconstruction, and the RoPE angle table.
//
// iS-KV summary, "Architecture Overview": the most recent tokens stay exact; "Reconstruction and
// Storage": compressed row i is (U Sigma B^T)[i] = (C B^T)[i], other rows are the exact rows.
#include "iskv_internal.cuh"

namespace iskv {

// One CTA per (row of the chunk, unit); blockIdx.z = path. Copies 128 elements (16-byte vectors).
__global__ void append_kernel(AppendArgs a) {
    const int path = blockIdx.z;
    const int i = blockIdx.x;            // row within the chunk
    const int unit = a.unit0 + blockIdx.y;
    const long long pos = a.pos0 + i;
    const int slot = (int)(pos % a.R);
    const size_t esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const char *src = static_cast<const char *>(a.src[path]) +
                      ((size_t)blockIdx.y * a.m_total + a.row0 + i) * D * esz;
    char *dst = static_cast<char *>(a.ring[path]) + ((size_t)unit * a.R + slot) * D * esz;
    const int nvec = (int)(D * esz / 16);
    if (threadIdx.x < nvec)
        reinterpret_cast<uint4 *>(dst)[threadIdx.x] = reinterpret_cast<const uint4 *>(src)[threadIdx.x];
}

cudaError_t launch_append(const AppendArgs &a, int n_units, cudaStream_t s) {
    if (a.rows <= 0) return cudaSuccess;
    append_kernel<<<dim3(a.rows, n_units, 2), 32, 0, s>>>(a);
    return cudaGetLastError();
}

// (cos, sin) of pos * theta^(-2j/d) for every position and pair j, computed in double and
// rounded once to float (the angle of a far position is too large for a float product).
__global__ void rope_table_kernel(float2 *table, long long max_tokens, double theta) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= max_tokens * DH) return;
    const long long pos = idx / DH;
    const int j = (int)(idx % DH);
    const double omega = pow(theta, -2.0 * j / (double)D);
    double sn, cs;
    sincos((double)pos * omega, &sn, &cs);
    table[idx] = make_float2((float)cs, (float)sn);
}

// Transposed copy for the tensor-core decode: table_t[q][pos] = (cos_2q, cos_2q+1, sin_2q,
// sin_2q+1) of pairs 2q and 2q+1 at position pos, so that the 32 rows of a warp read 32
// consecutive float4 (one coalesced line) instead of 32 rows 512 bytes apart, and the two cosines
// (sines) form one packed fp32 operand.
__global__ void rope_table_t_kernel(float4 *table_t, long long max_tokens, double theta) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= max_tokens * (DH / 2)) return;
    const int q = (int)(idx / max_tokens);
    const long long pos = idx % max_tokens;
    double s0, c0, s1, c1;
    sincos((double)pos * pow(theta, -2.0 * (2 * q) / (double)D), &s0, &c0);
    sincos((double)pos * pow(theta, -2.0 * (2 * q + 1) / (double)D), &s1, &c1);
    table_t[idx] = make_float4((float)c0, (float)c1, (float)s0, (float)s1);
}

cudaError_t launch_rope_table_t(float4 *table_t, long long max_tokens, double theta,
                                cudaStream_t s) {
    const long long n = max_tokens * (DH / 2);
    rope_table_t_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(table_t, max_tokens, theta);
    return cudaGetLastError();
}

cudaError_t launch_rope_table(float2 *table, long long max_tokens, double theta, cudaStream_t s) {
    const long long n = max_tokens * DH;
    const unsigned grid = (unsigned)((n + 255) / 256);
    rope_table_kernel<<<grid, 256, 0, s>>>(table, max_tokens, theta);
    return cudaGetLastError();
}

// One CTA per (tile of 64 positions, unit); 128 threads (one per channel).
__global__ void reconstruct_kernel(ReconArgs a) {
    extern __shared__ float sB[];        // basis row j, column c at [j * ks + c]
    const int unit = blockIdx.y;
    const int j = threadIdx.x;
    const int k = a.k, r = a.r, ks = k | 1;
    const float *B = a.basis + (size_t)unit * D * r;
    for (int o = threadIdx.x; o < D * k; o += blockDim.x) sB[(o / k) * ks + o % k] = B[(size_t)(o / k) * r + o % k];
    __syncthreads();
    const long long p0 = (long long)blockIdx.x * 64;
    for (int i = 0; i < 64; ++i) {
        const long long pos = p0 + i;
        if (pos >= a.t) break;
        float x;
        const bool protd = pos < a.n_c && a.pflags != nullptr &&
                           (a.pflags[(size_t)unit * a.fstride + pos] & a.fbit);
        if (protd) {
            // a protected position: the exact row from the path's store
            const int *pp = a.ppos + (size_t)unit * a.pcap;
            int lo = 0, hi = a.pcount[unit];
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (pp[mid] < pos) lo = mid + 1;
                else hi = mid;
            }
            x = (lo < a.pcount[unit] && pp[lo] == pos)
                    ? load_row_elem(a.pstore, ((size_t)unit * a.pcap + lo) * D + j, a.kv_dtype)
                    : 0.f;
        } else if (pos < a.n_c) {
            const size_t ci = ((size_t)coord_unit(unit, a.cdiv) * a.n_max + pos) * r;
            float s = 0.f;
            for (int l = 0; l < k; ++l) s = fmaf(load_coord(a.coords, ci + l, a.cbf), sB[j * ks + l], s);
            x = s;
        } else {
            const int slot = (int)(pos % a.R);
            x = load_row_elem(a.ring, ((size_t)unit * a.R + slot) * D + j, a.kv_dtype);
        }
        float *o = a.out + ((size_t)unit * a.t + pos) * D;
        if (a.apply_rope) {
            // pair (j, j + 64) lives in two threads: exchange through shared memory
            __shared__ float sx[D];
            sx[j] = x;
            __syncthreads();
            const float2 cs = a.rope_cs[pos * DH + (j & (DH - 1))];
            x = (j < DH) ? x * cs.x - sx[j + DH] * cs.y : x * cs.x + sx[j - DH] * cs.y;
            __syncthreads();
        }
        o[j] = x;
    }
}

cudaError_t launch_reconstruct(const ReconArgs &a, int n_units, cudaStream_t s) {
    if (a.t <= 0) return cudaSuccess;
    const size_t smem = (size_t)D * ((a.k | 1)) * sizeof(float);
    static size_t attr[64] = {0};
    const cudaError_t e = ensure_smem((const void *)reconstruct_kernel, smem, attr);
    if (e != cudaSuccess) return e;
    const unsigned gx = (unsigned)((a.t + 63) / 64);
    reconstruct_kernel<<<dim3(gx, n_units), D, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace iskv

namespace iskv {

// bf16 coordinates -> fp32 (the inspection copy of iskv_get_factors).
__global__ void coords_to_f32_kernel(float *dst, const __nv_bfloat16 *src, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        dst[i] = __bfloat162float(src[i]);
}

cudaError_t launch_coords_to_f32(float *dst, const void *src, size_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    coords_to_f32_kernel<<<grid, 256, 0, s>>>(dst, static_cast<const __nv_bfloat16 *>(src), n);
    return cudaGetLastError();
}

}  // namespace iskv
