// Decode attention with tensor-core key reconstruction (sm_100a tcgen05 + TMA).
//
// iS-KV summary, "Reconstruction and Storage": compressed rows are (C B^T)[i]; keys were
// compressed before RoPE, so a key tile K~ = C_K[tile] B_K^T (128 rows x 128 channels) is formed on
// the tensor cores and rotated afterwards, row by row.
//
// Split kernel: one CTA (8 warps) serves one split of one kv-head. Row i of a 128-row tile is TMEM
// lane i of the accumulator; warps w and w + 4 both read lanes 32 (w mod 4) .. +31 and take half of
// the RoPE channel pairs (j, j + 64) each, so every row has two threads. Per compressed tile: a
// TMA load of the key-coordinate tile (128-byte swizzle, 32 fp32 per row and K-block) and a bulk
// load of the value coordinates; the key coordinates are split into tf32 hi + lo parts and three
// kind::tf32 MMAs (hi*hi + hi*lo + lo*hi) give fp32-level keys in TMEM; the epilogue rotates the
// row at its position, forms the dot products with the G pre-scaled queries, updates the online
// softmax and accumulates sum_i p_i C_V[i] in rank space. The next tile's key coordinates are
// loaded while this tile's epilogue runs, its value coordinates while the softmax runs. Window
// tiles read the exact bf16/fp32 rows instead. Each split writes (max, sum, accumulator) partials.
//
// Merge kernel: one CTA per (q-head, kv-head) combines the splits (log-sum-exp weights) and
// expands the rank-space value sum once through B_V^T. It is launched as a programmatic dependent
// of the split kernel, so its prologue (staging B_V) overlaps the split kernel's tail.
#include <math_constants.h>

#include "iskv_internal.cuh"
#include "tc_util.cuh"

namespace iskv {

constexpr int TC_THREADS = 256;
constexpr int MERGE_THREADS = 128;
constexpr int MERGE_REG = 48;             // splits whose partials a merge thread keeps in registers
constexpr int KBLK_BYTES = 128 * 128;     // one K-block: 128 rows x 32 fp32

struct TcLayout {
    uint32_t b_hi, b_lo, a_hi, a_lo, v, q, x, red, bars, total;
};

// Shared-memory plan of the split kernel. Window tiles stage their exact value rows from a_hi
// onwards (a_hi, a_lo and v are contiguous and unused by window tiles otherwise).
__host__ __device__ inline TcLayout tc_layout(int kblocks, int rV, int esz, int G) {
    TcLayout L;
    uint32_t o = 0;
    L.b_hi = o; o += kblocks * KBLK_BYTES;
    L.b_lo = o; o += kblocks * KBLK_BYTES;
    L.a_hi = o; o += kblocks * KBLK_BYTES;
    L.a_lo = o; o += kblocks * KBLK_BYTES;
    L.v = o;
    const uint32_t vcomp = 128u * rV * 4u;
    const uint32_t vwin = 128u * D * esz;
    const uint32_t span = 2u * kblocks * KBLK_BYTES;      // a_hi + a_lo
    const int nq = (rV + 3) / 4, nqp = nq <= 8 ? 8 : nq <= 16 ? 16 : 32;
    const uint32_t redv = 8u * G * nqp * 16u;             // value-sum reduction in the stage
    uint32_t vb = vcomp > redv ? vcomp : redv;
    if (vwin > span + vb) vb = vwin - span;
    if (8u * G * 32u * 16u > span + vb) vb = 8u * G * 32u * 16u - span;   // window reduction
    o += (vb + 1023) & ~1023u;
    L.q = o; o += G * D * 4;
    L.x = o; o += 2 * G * 128 * 4;           // score halves, then (aliased) probabilities
    L.red = o; o += 2 * 4 * GMAX * 4;
    L.bars = o; o += 64;
    L.total = o + 1024;                    // slack for aligning the base to 1024 bytes
    return L;
}

size_t tc_smem_bytes(int kblocks, int rV, int esz, int G) {
    return tc_layout(kblocks, rV, esz, G).total;
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Split fp32 values into a tf32 "hi" part (top 19 bits, exact in tf32) kept in place and the
// exact remainder "lo" written at the same offset of the second buffer.
__device__ __forceinline__ void split_tf32(uint8_t *hi, uint8_t *lo, int bytes) {
    float4 *h4 = reinterpret_cast<float4 *>(hi);
    float4 *l4 = reinterpret_cast<float4 *>(lo);
    for (int i = threadIdx.x; i < bytes / 16; i += TC_THREADS) {
        float4 x = h4[i], h, l;
        h.x = __uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u);
        h.y = __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u);
        h.z = __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u);
        h.w = __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u);
        l.x = x.x - h.x;
        l.y = x.y - h.y;
        l.z = x.z - h.z;
        l.w = x.w - h.w;
        h4[i] = h;
        l4[i] = l;
    }
}

// 16 consecutive channels of an exact row (bf16 or fp32) as fp32.
__device__ __forceinline__ void load_row16(const void *ring, size_t base, int kv_dtype,
                                           float (&v)[16]) {
    if (kv_dtype == ISKV_BF16) {
        const uint4 *p = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const __nv_bfloat16 *>(ring) + base);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 u = p[q];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                v[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
                v[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(ring) + base);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = p[q];
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
    }
}

// Four consecutive channels of a value row staged in shared memory.
__device__ __forceinline__ float4 load_v4(const uint8_t *row, int c, int fmt) {
    if (fmt == 2) {                                   // bf16 row
        const uint2 u = *reinterpret_cast<const uint2 *>(row + 2 * c);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    return *reinterpret_cast<const float4 *>(row + 4 * c);
}

template <int GT>
__global__ void __launch_bounds__(TC_THREADS, 2) decode_tc_kernel(
    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmB,
    DecodeArgs a, TcExtra x) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int G = a.G, rV = a.r[1], kV = a.k[1];
    const int esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const TcLayout L = tc_layout(x.kblocks, rV, esz, G);
    uint8_t *bBh = sm + L.b_hi, *bBl = sm + L.b_lo, *bAh = sm + L.a_hi, *bAl = sm + L.a_lo;
    float *sQ = reinterpret_cast<float *>(sm + L.q);
    float *sX = reinterpret_cast<float *>(sm + L.x);            // [2 halves][G][128]
    float *sP = sX;                                             // [128][GT] (after the scores)
    float *sRed = reinterpret_cast<float *>(sm + L.red);        // [2][4][GMAX]
    uint64_t *bar_a = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *bar_v = bar_a + 1;
    uint64_t *bar_mma = bar_a + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_a + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, half = warp >> 2;
    // one-dimensional grid: all window splits first (short), then the compressed splits, so the
    // long compressed CTAs start in the first wave
    int ul, split;
    {
        const int nsw = a.n_split - a.n_split_c;
        const int W = (int)(gridDim.x / a.n_split) * nsw;
        int idx = blockIdx.x;
        if (idx < W) {
            ul = idx / nsw;
            split = a.n_split_c + idx % nsw;
        } else {
            idx -= W;
            ul = idx / a.n_split_c;
            split = idx % a.n_split_c;
        }
    }
    const int seq = ul / a.H, h = ul % a.H;
    const bool comp = split < a.n_split_c;
    uint8_t *bV = comp ? sm + L.v : bAh;                        // value rows of the tile
    const int vfmt = comp ? 4 : esz;
    const int vld = comp ? rV * 4 : D * esz;                    // bytes per staged value row
    const int nacc = comp ? kV : D;
    long long p0, p1;
    if (comp) {
        p0 = (long long)split * a.split_rows;
        p1 = min(a.n_c, p0 + a.split_rows);
    } else {
        p0 = a.n_c + (long long)(split - a.n_split_c) * DEC_TILE;
        p1 = min(a.t, p0 + DEC_TILE);
    }

    const size_t ring_base = (size_t)ul * a.R * D;
    const long long cu = coord_unit(ul, a.cdiv);   // the kv-head's coordinate unit
    const float *Cv = static_cast<const float *>(a.coords[1]) + (size_t)cu * a.n_max * rV;
    const uint32_t idesc = idesc_tf32(128, 128);
    const uint32_t abytes = x.kblocks * KBLK_BYTES;

    // thread 0: key-coordinate tile (TMA) and value rows (bulk copies) of the tile at t0; each
    // barrier phase gets exactly one arrival, which posts all bytes of that phase
    auto tma_a = [&](long long t0) {
        for (int kb = 0; kb < x.kblocks; ++kb)
            tma_load_2d(bAh + kb * KBLK_BYTES, &tmC, kb * 32,
                        (int)(x.row0 + (long long)cu * a.n_max + t0), bar_a);
    };
    auto issue_v = [&](long long t0, int rows) {
        if (comp) {
            mbar_arrive_expect_tx(bar_v, (uint32_t)rows * rV * 4);
            bulk_load(bV, Cv + (size_t)t0 * rV, (uint32_t)rows * rV * 4, bar_v);
        } else {
            const int s0 = (int)(t0 % a.R);
            const int n1 = min(rows, a.R - s0);
            const uint32_t rb = D * esz;
            const char *ring = static_cast<const char *>(a.ring[1]);
            mbar_arrive_expect_tx(bar_v, (uint32_t)rows * rb);
            bulk_load(bV, ring + (ring_base + (size_t)s0 * D) * esz, (uint32_t)n1 * rb, bar_v);
            if (n1 < rows)
                bulk_load(bV + (size_t)n1 * rb, ring + ring_base * esz, (uint32_t)(rows - n1) * rb,
                          bar_v);
        }
    };

    if (comp && warp == 0) tmem_alloc(tmem_slot, 256);
    // everything the previous kernel in the stream writes (rows, factors, queries) is read only
    // after this point; dependents may start once every CTA got here
    griddep_wait();
    griddep_launch_dependents();
    // outstanding phases (the same in every thread: issue conditions are uniform)
    bool pend_a = comp && p0 < p1, pend_v = p0 < p1, pend_m = false;
    uint32_t ph_a = 0, ph_v = 0, ph_m = 0;
    if (tid == 0) {
        mbar_init(bar_a, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        if (p0 < p1) {
            if (comp) {
                // the queries of this kv-head ride on the first key-tile barrier
                mbar_arrive_expect_tx(bar_a, 2 * abytes + (uint32_t)(G * D * 4));
                bulk_load(sQ, a.q + ((size_t)seq * a.H * G + (size_t)h * G) * D,
                          (uint32_t)(G * D * 4), bar_a);
                for (int kb = 0; kb < x.kblocks; ++kb)
                    tma_load_2d(bBh + kb * KBLK_BYTES, &tmB, kb * 32, x.brow0 + ul * D, bar_a);
                tma_a(p0);
            }
            issue_v(p0, (int)min((long long)DEC_TILE, p1 - p0));
        }
    }
    {
        // window CTAs load the queries through registers (compressed CTAs got them by bulk copy)
        const float4 *q4 = reinterpret_cast<const float4 *>(a.q + ((size_t)seq * a.H * G + (size_t)h * G) * D);
        float4 *s4 = reinterpret_cast<float4 *>(sQ);
        if (!comp && tid < G * D / 4) s4[tid] = q4[tid];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = comp ? *tmem_slot : 0u;
    bool ok = true;

    float mrun[GT], lrun[GT];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
        mrun[g] = -CUDART_INF_F;
        lrun[g] = 0.f;
    }
    const int row = 32 * wq + lane;
    const int jb = 32 * half;                   // this thread's first channel pair
    // value sums in rank space (or channels, window CTAs): thread = (channel quad qd, row slice
    // sl); each thread keeps its slice's sums in registers over all tiles of the split, rescaled
    // with the running max, and the slices are added once at the end
    const int nq = (nacc + 3) >> 2;
    const int nqp = nq <= 8 ? 8 : nq <= 16 ? 16 : 32;
    const int nsl = TC_THREADS / nqp;
    const int qd = tid & (nqp - 1), sl = tid / nqp;
    float4 vacc[GT];
#pragma unroll
    for (int g = 0; g < GT; ++g) vacc[g] = make_float4(0.f, 0.f, 0.f, 0.f);

    // thread 0 issues the three-term tf32 product of the staged key-coordinate tile into TMEM
    // accumulator `buf` (columns 128 buf .. 128 buf + 127)
    auto issue_mma = [&](int buf) {
        tc_fence_after();
        const uint32_t aH = smem_u32(bAh), aL = smem_u32(bAl);
        const uint32_t bH = smem_u32(bBh), bL = smem_u32(bBl);
        const uint32_t d = tmem + 128u * buf;
        uint32_t acc = 0;
        for (int kb = 0; kb < x.kblocks; ++kb)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t off = kb * KBLK_BYTES + kk * 32;
                mma_tf32(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bH + off), idesc, acc);
                acc = 1;
                mma_tf32(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bL + off), idesc, 1);
                mma_tf32(d, sw128_kmajor_desc(aL + off), sw128_kmajor_desc(bH + off), idesc, 1);
            }
        mma_commit(bar_mma);
    };

    // first compressed tile: split B and A, start its product
    if (comp && p0 < p1) {
        ok = __syncthreads_and(mbar_wait(bar_a, ph_a)) != 0;
        if (ok) {
            pend_a = false;
            ph_a ^= 1;
            split_tf32(bBh, bBl, abytes);
            split_tf32(bAh, bAl, abytes);
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) issue_mma(0);
            pend_m = true;
        }
    }

    int it = 0;
    for (long long t0 = p0; t0 < p1 && ok; t0 += DEC_TILE, ++it) {
        const int rows = (int)min((long long)DEC_TILE, p1 - t0);
        const bool valid = row < rows;
        const long long pos = t0 + row;
        const bool rope = valid && x.rope_t != nullptr;
        const bool more = t0 + DEC_TILE < p1;
        float part[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) part[g] = 0.f;
        // RoPE angles of this thread's 32 pairs, first half now (under the MMA wait)
        float4 cs[16];
        // (transposed table: float4 q of this row is entry (jb/2 + q) * rope_rows + pos)
        const float4 *c4 = x.rope_t + (size_t)(jb / 2) * x.rope_rows + pos;
        if (rope) {
#pragma unroll
            for (int q = 0; q < 8; ++q) cs[q] = c4[(size_t)q * x.rope_rows];
        }
        if (comp) {
            ok = __syncthreads_and(mbar_wait(bar_mma, ph_m)) != 0;
            tc_fence_after();
            if (!ok) break;
            pend_m = false;
            ph_m ^= 1;
            // the key-coordinate buffers are free again: fetch the next tile's under this epilogue
            if (more) {
                pend_a = true;
                if (tid == 0) {
                    mbar_arrive_expect_tx(bar_a, abytes);
                    tma_a(t0 + DEC_TILE);
                }
            }
        }

        // ---- this row's key, channel pairs (j, j + 64) for j in [jb, jb + 32), two chunks;
        //      RoPE and the dot products in packed fp32 pairs ----------------------------------
        const uint32_t trow = tmem + 128u * (it & 1) + ((uint32_t)(wq * 32) << 16);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            const int j0 = jb + 16 * ch;
            float lo[16], hi[16];
            if (comp) {
                tmem_ld16(trow + j0, lo);
                tmem_ld16(trow + 64 + j0, hi);
                tmem_wait_ld();
            } else if (valid) {
                const bool fresh = pos == a.new_pos;      // appended by this call
                const void *src = fresh ? a.new_row[0] : a.ring[0];
                const size_t rb = fresh ? (size_t)ul * D : ring_base + (size_t)(pos % a.R) * D;
                load_row16(src, rb + j0, a.kv_dtype, lo);
                load_row16(src, rb + 64 + j0, a.kv_dtype, hi);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) lo[j] = hi[j] = 0.f;
            }
            float2 L2[8], H2[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                L2[q] = make_float2(lo[2 * q], lo[2 * q + 1]);
                H2[q] = make_float2(hi[2 * q], hi[2 * q + 1]);
            }
            if (rope) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 w = cs[8 * ch + q];              // (cos, cos, sin, sin)
                    const float2 c = make_float2(w.x, w.y), sn = make_float2(w.z, w.w);
                    const float2 ys = __fmul2_rn(H2[q], sn), xs = __fmul2_rn(L2[q], sn);
                    const float2 xl = __ffma2_rn(L2[q], c, make_float2(-ys.x, -ys.y));
                    H2[q] = __ffma2_rn(H2[q], c, xs);
                    L2[q] = xl;
                }
                if (ch == 0) {                   // second half of the angles, under this chunk
#pragma unroll
                    for (int q = 8; q < 16; ++q) cs[q] = c4[(size_t)q * x.rope_rows];
                }
            }
#pragma unroll
            for (int g = 0; g < GT; ++g) {
                if (g < G) {
                    const float4 *ql = reinterpret_cast<const float4 *>(sQ + g * D + j0);
                    const float4 *qh = reinterpret_cast<const float4 *>(sQ + g * D + 64 + j0);
                    float2 s2 = make_float2(part[g], 0.f);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 u = ql[q], v = qh[q];
                        s2 = __ffma2_rn(make_float2(u.x, u.y), L2[2 * q], s2);
                        s2 = __ffma2_rn(make_float2(u.z, u.w), L2[2 * q + 1], s2);
                        s2 = __ffma2_rn(make_float2(v.x, v.y), H2[2 * q], s2);
                        s2 = __ffma2_rn(make_float2(v.z, v.w), H2[2 * q + 1], s2);
                    }
                    part[g] = s2.x + s2.y;
                }
            }
        }
        // ---- the two halves of each row meet; both threads hold the same score ------------------
#pragma unroll
        for (int g = 0; g < GT; ++g)
            if (g < G) sX[(half * G + g) * 128 + row] = part[g];
        __syncthreads();
#pragma unroll
        for (int g = 0; g < GT; ++g)
            if (g < G) {
                part[g] = (sX[g * 128 + row] + sX[(G + g) * 128 + row]) * a.scale;
                const float m = warp_max_f(valid ? part[g] : -CUDART_INF_F);
                if (half == 0 && lane == 0) sRed[wq * GMAX + g] = m;
            }
        // ---- next tile: split its key coordinates and start its product into the other
        //      accumulator, so the tensor cores work under this tile's softmax and values -------
        bool okn = true;
        if (comp && more) {
            okn = mbar_wait(bar_a, ph_a);
            if (okn) split_tf32(bAh, bAl, abytes);
            fence_proxy_async_smem();
        }
        ok = __syncthreads_and(okn) != 0;
        if (!ok) break;
        if (comp && more) {
            pend_a = false;
            ph_a ^= 1;
            if (tid == 0) issue_mma((it + 1) & 1);
            pend_m = true;
        }
        // ---- online softmax: every thread keeps the same running max and sum -------------------
        float alpha[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) {
            alpha[g] = 1.f;
            if (g < G) {
                const float mt = fmaxf(fmaxf(sRed[g], sRed[GMAX + g]),
                                       fmaxf(sRed[2 * GMAX + g], sRed[3 * GMAX + g]));
                const float m_new = fmaxf(mrun[g], mt);
                const float pr = valid ? expf(part[g] - m_new) : 0.f;
                if ((g & 1) == half) {
                    sP[row * GT + g] = pr;
                    const float s = warp_sum_f(pr);
                    if (lane == 0) sRed[4 * GMAX + wq * GMAX + g] = s;
                }
                alpha[g] = expf(mrun[g] - m_new);
                mrun[g] = m_new;
            }
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < GT; ++g)
            if (g < G) {
                const float s = (sRed[4 * GMAX + g] + sRed[5 * GMAX + g]) +
                                (sRed[6 * GMAX + g] + sRed[7 * GMAX + g]);
                lrun[g] = fmaf(lrun[g], alpha[g], s);
            }
        // ---- value accumulation: vacc_g = vacc_g * alpha_g + sum_i p[g][i] V[i][quad] ------------
        // quads vary fastest across a warp's lanes, so the lanes of a shared-memory phase read
        // consecutive 16-byte (8-byte for bf16) pieces of one staged row (no bank conflicts);
        // slice sl takes rows sl, sl + nsl, ... Quads past the row's end (nqp is a power of two)
        // read the next row's values and are never used.
        ok = __syncthreads_and(mbar_wait(bar_v, ph_v)) != 0;
        if (!ok) break;
        pend_v = false;
        ph_v ^= 1;
        if (!comp && a.new_pos >= t0 && a.new_pos < t0 + rows) {
            // fused append: the staged copy of this slot is stale; take the caller's row and
            // store K and V in the ring for later calls (one CTA owns this position)
            const int i = (int)(a.new_pos - t0);
            const size_t slot = ring_base + (size_t)(a.new_pos % a.R) * D;
            if (a.kv_dtype == ISKV_BF16) {
                const __nv_bfloat16 *nk = static_cast<const __nv_bfloat16 *>(a.new_row[0]) + (size_t)ul * D;
                const __nv_bfloat16 *nv = static_cast<const __nv_bfloat16 *>(a.new_row[1]) + (size_t)ul * D;
                __nv_bfloat16 *rk = const_cast<__nv_bfloat16 *>(static_cast<const __nv_bfloat16 *>(a.ring[0])) + slot;
                __nv_bfloat16 *rv = const_cast<__nv_bfloat16 *>(static_cast<const __nv_bfloat16 *>(a.ring[1])) + slot;
                if (tid < D) {
                    const __nv_bfloat16 v = nv[tid];
                    reinterpret_cast<__nv_bfloat16 *>(bV + (size_t)i * vld)[tid] = v;
                    rv[tid] = v;
                    rk[tid] = nk[tid];
                }
            } else {
                const float *nk = static_cast<const float *>(a.new_row[0]) + (size_t)ul * D;
                const float *nv = static_cast<const float *>(a.new_row[1]) + (size_t)ul * D;
                float *rk = const_cast<float *>(static_cast<const float *>(a.ring[0])) + slot;
                float *rv = const_cast<float *>(static_cast<const float *>(a.ring[1])) + slot;
                if (tid < D) {
                    const float v = nv[tid];
                    reinterpret_cast<float *>(bV + (size_t)i * vld)[tid] = v;
                    rv[tid] = v;
                    rk[tid] = nk[tid];
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int g = 0; g < GT; ++g)
            if (g < G) {
                const float2 al2 = make_float2(alpha[g], alpha[g]);
                const float2 a01 = __fmul2_rn(al2, make_float2(vacc[g].x, vacc[g].y));
                const float2 a23 = __fmul2_rn(al2, make_float2(vacc[g].z, vacc[g].w));
                vacc[g] = make_float4(a01.x, a01.y, a23.x, a23.y);
            }
#pragma unroll 4
        for (int i = sl; i < rows; i += nsl) {
            const float4 v = load_v4(bV + (size_t)i * vld, 4 * qd, vfmt);
            const float2 v01 = make_float2(v.x, v.y), v23 = make_float2(v.z, v.w);
            float pv[GT];                       // this row's probabilities, one vector load
            if (GT >= 4) {
#pragma unroll
                for (int g4 = 0; g4 < GT / 4; ++g4) {
                    const float4 p4 = reinterpret_cast<const float4 *>(sP + i * GT)[g4];
                    pv[4 * g4] = p4.x;
                    pv[4 * g4 + 1] = p4.y;
                    pv[4 * g4 + 2] = p4.z;
                    pv[4 * g4 + 3] = p4.w;
                }
            } else {
#pragma unroll
                for (int g = 0; g < GT; ++g) pv[g] = sP[i * GT + g];
            }
#pragma unroll
            for (int g = 0; g < GT; ++g)
                if (g < G) {
                    const float pg = pv[g];
                    const float2 p2 = make_float2(pg, pg);
                    const float2 a01 = __ffma2_rn(p2, v01, make_float2(vacc[g].x, vacc[g].y));
                    const float2 a23 = __ffma2_rn(p2, v23, make_float2(vacc[g].z, vacc[g].w));
                    vacc[g] = make_float4(a01.x, a01.y, a23.x, a23.y);
                }
        }
        fence_proxy_async_smem();              // the stage was written through the generic proxy
        tc_fence_before();
        __syncthreads();                       // value rows, probabilities and TMEM consumed
        if (more) {
            pend_v = true;
            if (tid == 0) issue_v(t0 + DEC_TILE, (int)min((long long)DEC_TILE, p1 - t0 - DEC_TILE));
        }
    }
    if (!ok && tid == 0) {
        // a wait gave up: record it, then let this CTA's own copies and MMAs drain (bounded)
        set_status(x.status, ISKV_ERR_TIMEOUT);
        if (pend_a) mbar_wait(bar_a, ph_a);
        if (pend_v) mbar_wait(bar_v, ph_v);
        if (pend_m) mbar_wait(bar_mma, ph_m);
    }

    // ---- the slices' value sums meet once: within the warp (shuffles), then across the 8 warps
    //      in the value stage (free: every copy into it has completed or drained) -------------------
#pragma unroll
    for (int g = 0; g < GT; ++g)
        if (g < G) {
            for (int o = nqp; o < 32; o <<= 1) {
                vacc[g].x += __shfl_xor_sync(0xffffffffu, vacc[g].x, o);
                vacc[g].y += __shfl_xor_sync(0xffffffffu, vacc[g].y, o);
                vacc[g].z += __shfl_xor_sync(0xffffffffu, vacc[g].z, o);
                vacc[g].w += __shfl_xor_sync(0xffffffffu, vacc[g].w, o);
            }
        }
    float *sRedV = reinterpret_cast<float *>(bV);               // [8 warps][G][4 nqp]
    __syncthreads();
    if (lane < nqp) {
#pragma unroll
        for (int g = 0; g < GT; ++g)
            if (g < G) reinterpret_cast<float4 *>(sRedV)[(warp * G + g) * nqp + qd] = vacc[g];
    }
    __syncthreads();

    // ---- partials: [m, l, acc[nacc]] per q-head ---------------------------------------------------
    float *ws = a.ws + ((size_t)ul * a.max_splits + split) * G * (2 + D);
    for (int o = tid; o < G * nacc; o += TC_THREADS) {
        const int g = o / nacc, c = o % nacc;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += sRedV[((w * G + g) * nqp) * 4 + c];
        ws[g * (2 + D) + 2 + c] = sum;
    }
    if (tid < G) {
#pragma unroll
        for (int g = 0; g < GT; ++g)
            if (g == tid) {
                ws[g * (2 + D)] = mrun[g];
                ws[g * (2 + D) + 1] = lrun[g];
            }
    }

    // ---- release tensor memory -------------------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (comp && warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// One CTA per (q-head g, kv-head unit): log-sum-exp merge of the splits and the expansion of the
// rank-space value sum through B_V^T. Thread j owns output channel j.
__global__ void __launch_bounds__(MERGE_THREADS) decode_merge_kernel(DecodeArgs a) {
    extern __shared__ float msm[];
    const int G = a.G, rV = a.r[1], kV = a.k[1];
    const int ldb = kV | 1;
    float *sBV = msm;                                   // [D][ldb]
    float *sW = sBV + D * ldb;                          // [max_splits] maxima, then weights
    float *sL = sW + a.max_splits;                      // [max_splits] sums
    float *sAcc = sL + a.max_splits;                    // [D]
    float *sRed = sAcc + D;                             // [8]
    const int g = blockIdx.x, ul = blockIdx.y;
    const int seq = ul / a.H, h = ul % a.H;
    const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
    // the next kernel in the stream (the next decode's split kernel) may start its prologue
    // now; it reads nothing this kernel writes before its own dependency wait
    griddep_launch_dependents();
    // B_V was written before the split kernel started: stage it while the splits finish
    const float *B = a.basis[1] + (size_t)ul * D * rV;
    for (int o = j; o < D * kV; o += MERGE_THREADS) sBV[(o / kV) * ldb + o % kV] = B[(size_t)(o / kV) * rV + o % kV];
    griddep_wait();

    // every load this thread needs is issued at once: the maxima and sums of splits j, j + 128,
    // ... and its channel of the first MERGE_REG splits (one L2 round trip)
    const int ns = a.n_split, nsc = a.n_split_c;
    const size_t stride = (size_t)G * (2 + D);
    const float *wsu = a.ws + (size_t)ul * a.max_splits * stride + (size_t)g * (2 + D);
    const float *col = wsu + 2 + j;
    float v[MERGE_REG];
#pragma unroll
    for (int u = 0; u < MERGE_REG; ++u)
        v[u] = (u < ns && (u >= nsc || j < kV)) ? __ldcg(col + u * stride) : 0.f;
    float m = -CUDART_INF_F;
    for (int s = j; s < ns; s += MERGE_THREADS) {
        const float ms = __ldcg(wsu + s * stride);
        sW[s] = ms;
        sL[s] = __ldcg(wsu + s * stride + 1);
        m = fmaxf(m, ms);
    }
    m = warp_max_f(m);
    if (lane == 0) sRed[warp] = m;
    __syncthreads();
    const float M = fmaxf(fmaxf(sRed[0], sRed[1]), fmaxf(sRed[2], sRed[3]));
    float l = 0.f;
    for (int s = j; s < ns; s += MERGE_THREADS) {
        const float w = expf(sW[s] - M);
        sW[s] = w;
        l = fmaf(w, sL[s], l);
    }
    l = warp_sum_f(l);
    if (lane == 0) sRed[4 + warp] = l;
    __syncthreads();
    const float lsum = (sRed[4] + sRed[5]) + (sRed[6] + sRed[7]);

    float accr = 0.f, accw = 0.f;
#pragma unroll
    for (int u = 0; u < MERGE_REG; ++u)
        if (u < ns) {
            if (u < nsc) accr = fmaf(sW[u], v[u], accr);
            else accw = fmaf(sW[u], v[u], accw);
        }
    for (int s = MERGE_REG; s < ns; ++s) {
        if (s < nsc) {
            if (j < kV) accr = fmaf(sW[s], __ldcg(col + s * stride), accr);
        } else {
            accw = fmaf(sW[s], __ldcg(col + s * stride), accw);
        }
    }
    sAcc[j] = accr;
    __syncthreads();
    float o = accw;
    const float *br = sBV + j * ldb;
    for (int c = 0; c < kV; ++c) o = fmaf(sAcc[c], br[c], o);
    a.out[((size_t)seq * a.H * G + (size_t)h * G + g) * D + j] = o / lsum;
}

size_t merge_smem_bytes(int kV, int max_splits) {
    return ((size_t)D * (kV | 1) + 2 * (size_t)max_splits + D + 8) * sizeof(float);
}

cudaError_t launch_decode_tc(const CUtensorMap *tmC, const CUtensorMap *tmB, const DecodeArgs &a,
                             const TcExtra &x, int n_units, cudaStream_t s) {
    const int esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const size_t smem = tc_smem_bytes(x.kblocks, a.r[1], esz, a.G);
    const size_t msmem = merge_smem_bytes(a.k[1], a.max_splits);
    // opt-in dynamic shared memory, raised per device whenever a launch needs more
    static size_t attr_tc[64] = {0}, attr_merge[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (smem > attr_tc[dev]) {
        const void *fns[4] = {(const void *)decode_tc_kernel<1>, (const void *)decode_tc_kernel<2>,
                              (const void *)decode_tc_kernel<4>, (const void *)decode_tc_kernel<8>};
        for (const void *f : fns) {
            e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        attr_tc[dev] = smem;
    }
    if (msmem > attr_merge[dev]) {
        e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)msmem);
        if (e != cudaSuccess) return e;
        attr_merge[dev] = msmem;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_split * n_units);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (a.G <= 1 ? 1 : a.G <= 2 ? 2 : a.G <= 4 ? 4 : 8) {
    case 1: e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<1>, *tmC, *tmB, a, x); break;
    case 2: e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<2>, *tmC, *tmB, a, x); break;
    case 4: e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<4>, *tmC, *tmB, a, x); break;
    default: e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<8>, *tmC, *tmB, a, x); break;
    }
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(a.G, n_units);
    cfg.blockDim = dim3(MERGE_THREADS);
    cfg.dynamicSmemBytes = msmem;
    return cudaLaunchKernelEx(&cfg, decode_merge_kernel, a);
}

}  // namespace iskv
