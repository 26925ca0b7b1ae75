// Decode attention with tensor-core key reconstruction (sm_100a tcgen05 + TMA).
//
// iS-KV summary, "Reconstruction and Storage": compressed rows are (C B^T)[i]; keys were
// compressed before RoPE, so a key tile K~ = C_K[tile] B_K^T (128 rows x 128 channels) is formed on
// the tensor cores and rotated afterwards, row by row. One CTA (4 warps) serves one split of one
// kv-head; thread i owns row i of the tile, which is TMEM lane i of the accumulator.
//
// Per compressed tile: a TMA load of the coordinate tile (128-byte swizzle, 32 fp32 per row and
// K-block) and a bulk load of the value coordinates; the key coordinates are split into tf32
// hi + lo parts in place and three kind::tf32 MMAs (hi*hi + hi*lo + lo*hi) give fp32-level keys in
// TMEM; the epilogue reads the row (tcgen05.ld), applies RoPE at the row's position, takes the dot
// products with the G pre-scaled queries, updates the online softmax and accumulates
// sum_i p_i C_V[i] in rank space. Window tiles read the exact bf16/fp32 rows instead.
// The last CTA of a kv-head to finish merges all splits (log-sum-exp) and expands the rank-space
// value sum once through B_V^T; an arrival counter, reset by that CTA, decides who is last, so no
// CTA ever waits for another.
#include <math_constants.h>

#include "iskv_internal.cuh"
#include "tc_util.cuh"

namespace iskv {

constexpr int TC_THREADS = 128;
constexpr int KBLK_BYTES = 128 * 128;     // one K-block: 128 rows x 32 fp32

struct TcLayout {
    uint32_t b_hi, b_lo, a_hi, a_lo, v, q, p, red, stat, bars, total;
};

__host__ __device__ inline TcLayout tc_layout(int kblocks, int rV, int esz) {
    TcLayout L;
    uint32_t o = 0;
    L.b_hi = o; o += kblocks * KBLK_BYTES;
    L.b_lo = o; o += kblocks * KBLK_BYTES;
    L.a_hi = o; o += kblocks * KBLK_BYTES;
    L.a_lo = o; o += kblocks * KBLK_BYTES;
    L.v = o;
    const uint32_t vb = (uint32_t)(128 * rV * 4) > (uint32_t)(128 * D * esz) ? 128 * rV * 4 : 128 * D * esz;
    o += (vb + 1023) & ~1023u;
    L.q = o; o += GMAX * D * 4;
    L.p = o; o += GMAX * 128 * 4;
    L.red = o; o += 2 * 4 * GMAX * 4;
    L.stat = o; o += 4 * GMAX * 4;
    L.bars = o; o += 64;
    L.total = o + 1024;                    // slack for aligning the base to 1024 bytes
    return L;
}

size_t tc_smem_bytes(int kblocks, int rV, int esz) { return tc_layout(kblocks, rV, esz).total; }

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

__device__ __forceinline__ void load_row32(const void *ring, size_t base, int kv_dtype,
                                           float (&v)[32]) {
    if (kv_dtype == ISKV_BF16) {
        const uint4 *p = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const __nv_bfloat16 *>(ring) + base);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
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
        for (int q = 0; q < 8; ++q) {
            const float4 f = p[q];
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
    }
}

__global__ void __launch_bounds__(TC_THREADS, 2) decode_tc_kernel(
    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmB,
    DecodeArgs a, TcExtra x) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int G = a.G, rV = a.r[1], kV = a.k[1];
    const int esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const TcLayout L = tc_layout(x.kblocks, rV, esz);
    uint8_t *bBh = sm + L.b_hi, *bBl = sm + L.b_lo, *bAh = sm + L.a_hi, *bAl = sm + L.a_lo;
    uint8_t *bV = sm + L.v;
    float *sQ = reinterpret_cast<float *>(sm + L.q);
    float *sP = reinterpret_cast<float *>(sm + L.p);
    float *sRed = reinterpret_cast<float *>(sm + L.red);        // [2][4 warps][GMAX]
    float *sM = reinterpret_cast<float *>(sm + L.stat);         // [GMAX] running max
    float *sL = sM + GMAX, *sAl = sL + GMAX;
    int *sFlag = reinterpret_cast<int *>(sAl + GMAX);
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *bar_mma = bar_load + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ul = blockIdx.y, split = blockIdx.x;
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
    {
        const float4 *q4 = reinterpret_cast<const float4 *>(a.q + ((size_t)seq * a.H * G + (size_t)h * G) * D);
        float4 *s4 = reinterpret_cast<float4 *>(sQ);
        const float sc = a.scale;
        float4 v[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int o = tid + TC_THREADS * u;
            v[u] = o < G * D / 4 ? q4[o] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int o = tid + TC_THREADS * u;
            if (o < G * D / 4) s4[o] = make_float4(v[u].x * sc, v[u].y * sc, v[u].z * sc, v[u].w * sc);
        }
    }
    if (tid < G) {
        sM[tid] = -CUDART_INF_F;
        sL[tid] = 0.f;
    }
    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (comp && warp == 0) tmem_alloc(tmem_slot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = comp ? *tmem_slot : 0u;
    uint32_t ph_load = 0, ph_mma = 0;
    bool ok = true;

    const size_t ring_base = (size_t)ul * a.R * D;
    const float *Cv = a.coords[1] + (size_t)ul * a.n_max * rV;
    const uint32_t idesc = idesc_tf32(128, 128);

    // thread 0: loads of one tile (key coordinates by TMA, value coordinates or exact window
    // value rows by bulk copy); the caller has posted the expected byte count
    auto issue_tile = [&](long long t0, int rows) {
        if (comp) {
            for (int kb = 0; kb < x.kblocks; ++kb)
                tma_load_2d(bAh + kb * KBLK_BYTES, &tmC, kb * 32,
                            (int)(x.row0 + (long long)ul * a.n_max + t0), bar_load);
            bulk_load(bV, Cv + (size_t)t0 * rV, (uint32_t)rows * rV * 4, bar_load);
        } else {
            const int s0 = (int)(t0 % a.R);
            const int n1 = min(rows, a.R - s0);
            const uint32_t rb = D * esz;
            const char *ring = static_cast<const char *>(a.ring[1]);
            bulk_load(bV, ring + (ring_base + (size_t)s0 * D) * esz, (uint32_t)n1 * rb, bar_load);
            if (n1 < rows)
                bulk_load(bV + (size_t)n1 * rb, ring + ring_base * esz, (uint32_t)(rows - n1) * rb,
                          bar_load);
        }
    };
    auto tile_bytes = [&](int rows) -> uint32_t {
        return comp ? x.kblocks * KBLK_BYTES + (uint32_t)rows * rV * 4 : (uint32_t)rows * D * esz;
    };
    if (tid == 0 && p0 < p1) {
        const int rows0 = (int)min((long long)DEC_TILE, p1 - p0);
        mbar_arrive_expect_tx(bar_load, tile_bytes(rows0) + (comp ? x.kblocks * KBLK_BYTES : 0u));
        if (comp)
            for (int kb = 0; kb < x.kblocks; ++kb)
                tma_load_2d(bBh + kb * KBLK_BYTES, &tmB, kb * 32, x.brow0 + ul * D, bar_load);
        issue_tile(p0, rows0);
    }

    float vacc[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) vacc[w] = 0.f;
    const int nacc = comp ? kV : D;

    for (long long t0 = p0; t0 < p1 && ok; t0 += DEC_TILE) {
        const int rows = (int)min((long long)DEC_TILE, p1 - t0);
        if (t0 != p0) {
            tc_fence_before();
            __syncthreads();                 // previous tile fully consumed (smem and TMEM)
            if (tid == 0) {
                mbar_arrive_expect_tx(bar_load, tile_bytes(rows));
                issue_tile(t0, rows);
            }
        }
        ok = __syncthreads_and(mbar_wait(bar_load, ph_load)) != 0;
        ph_load ^= 1;
        if (!ok) break;
        if (comp && t0 == p0) split_tf32(bBh, bBl, x.kblocks * KBLK_BYTES);

        const int row = tid;
        const bool valid = row < rows;
        const long long pos = t0 + row;
        const bool rope = valid && a.rope_cs != nullptr;
        float4 cs0[16];
        float part[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) part[g] = 0.f;

        if (comp) {
            split_tf32(bAh, bAl, x.kblocks * KBLK_BYTES);
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t aH = smem_u32(bAh), aL = smem_u32(bAl);
                const uint32_t bH = smem_u32(bBh), bL = smem_u32(bBl);
                uint32_t acc = 0;
                for (int kb = 0; kb < x.kblocks; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t off = kb * KBLK_BYTES + kk * 32;
                        mma_tf32(tmem, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bH + off), idesc, acc);
                        acc = 1;
                        mma_tf32(tmem, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bL + off), idesc, 1);
                        mma_tf32(tmem, sw128_kmajor_desc(aL + off), sw128_kmajor_desc(bH + off), idesc, 1);
                    }
                mma_commit(bar_mma);
            }
            if (rope) {                       // RoPE angles of pass 0 load while the MMA runs
                const float4 *cs = reinterpret_cast<const float4 *>(a.rope_cs + pos * DH);
#pragma unroll
                for (int q = 0; q < 16; ++q) cs0[q] = cs[q];
            }
            ok = __syncthreads_and(mbar_wait(bar_mma, ph_mma)) != 0;
            ph_mma ^= 1;
            tc_fence_after();
            if (!ok) break;
        }

        if (!comp && rope) {
            const float4 *cs = reinterpret_cast<const float4 *>(a.rope_cs + pos * DH);
#pragma unroll
            for (int q = 0; q < 16; ++q) cs0[q] = cs[q];
        }
        // ---- this row's key (two passes: channel pairs (j, j+64), j in [32hp, 32hp+32)) -------
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
            float lo[32], hi[32];
            if (comp) {
                tmem_ld32(trow + hp * 32, lo);
                tmem_ld32(trow + 64 + hp * 32, hi);
                tmem_wait_ld();
            } else if (valid) {
                const size_t rb = ring_base + (size_t)(pos % a.R) * D;
                load_row32(a.ring[0], rb + hp * 32, a.kv_dtype, lo);
                load_row32(a.ring[0], rb + 64 + hp * 32, a.kv_dtype, hi);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) lo[j] = hi[j] = 0.f;
            }
            if (rope) {
                const float4 *cs = reinterpret_cast<const float4 *>(a.rope_cs + pos * DH + hp * 32);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float4 w = hp == 0 ? cs0[q] : cs[q];
                    const float x0 = lo[2 * q], y0 = hi[2 * q], x1 = lo[2 * q + 1], y1 = hi[2 * q + 1];
                    lo[2 * q] = x0 * w.x - y0 * w.y;
                    hi[2 * q] = y0 * w.x + x0 * w.y;
                    lo[2 * q + 1] = x1 * w.z - y1 * w.w;
                    hi[2 * q + 1] = y1 * w.z + x1 * w.w;
                }
            }
#pragma unroll
            for (int g = 0; g < GMAX; ++g) {
                if (g < G) {
                    const float4 *ql = reinterpret_cast<const float4 *>(sQ + g * D + hp * 32);
                    const float4 *qh = reinterpret_cast<const float4 *>(sQ + g * D + 64 + hp * 32);
                    float s = part[g];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 u = ql[q], v = qh[q];
                        s = fmaf(u.x, lo[4 * q], s);
                        s = fmaf(u.y, lo[4 * q + 1], s);
                        s = fmaf(u.z, lo[4 * q + 2], s);
                        s = fmaf(u.w, lo[4 * q + 3], s);
                        s = fmaf(v.x, hi[4 * q], s);
                        s = fmaf(v.y, hi[4 * q + 1], s);
                        s = fmaf(v.z, hi[4 * q + 2], s);
                        s = fmaf(v.w, hi[4 * q + 3], s);
                    }
                    part[g] = s;
                }
            }
        }
        // ---- online softmax over the tile's rows -------------------------------------------------
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            if (g < G) {
                const float m = warp_max_f(valid ? part[g] : -CUDART_INF_F);
                if (lane == 0) sRed[warp * GMAX + g] = m;
            }
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            if (g < G) {
                float mt = sRed[g];
#pragma unroll
                for (int w = 1; w < 4; ++w) mt = fmaxf(mt, sRed[w * GMAX + g]);
                const float m_new = fmaxf(sM[g], mt);
                const float pr = valid ? expf(part[g] - m_new) : 0.f;
                sP[g * DEC_TILE + row] = pr;
                const float s = warp_sum_f(pr);
                if (lane == 0) sRed[4 * GMAX + warp * GMAX + g] = s;
                part[g] = m_new;                 // keep m_new for the stats update
            }
        }
        __syncthreads();
        if (tid < G) {
            const int g = tid;
            const float m_new = part[g];
            const float alpha = expf(sM[g] - m_new);
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) s += sRed[4 * GMAX + w * GMAX + g];
            sL[g] = sL[g] * alpha + s;
            sM[g] = m_new;
            sAl[g] = alpha;
        }
        __syncthreads();
        // ---- value accumulation: acc[g][c] = acc * alpha_g + sum_i p[g][i] V[i][c] ------------------
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const int o = tid + TC_THREADS * w;
            if (o < G * nacc) {
                const int g = o / nacc, c = o % nacc;
                const float *pg = sP + g * DEC_TILE;
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
                const int ld = comp ? rV : D;
                int i = 0;
                if (comp || esz == 4) {
                    const float *vv = reinterpret_cast<const float *>(bV) + c;
                    for (; i + 3 < rows; i += 4)
#pragma unroll
                        for (int u = 0; u < 4; ++u) s4[u] = fmaf(pg[i + u], vv[(i + u) * ld], s4[u]);
                    for (; i < rows; ++i) s4[0] = fmaf(pg[i], vv[i * ld], s4[0]);
                } else {
                    const __nv_bfloat16 *vv = reinterpret_cast<const __nv_bfloat16 *>(bV) + c;
                    for (; i + 3 < rows; i += 4)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            s4[u] = fmaf(pg[i + u], __bfloat162float(vv[(i + u) * D]), s4[u]);
                    for (; i < rows; ++i) s4[0] = fmaf(pg[i], __bfloat162float(vv[i * D]), s4[0]);
                }
                vacc[w] = fmaf(vacc[w], sAl[g], (s4[0] + s4[1]) + (s4[2] + s4[3]));
            }
        }
    }
    if (!ok && tid == 0) set_status(x.status, ISKV_ERR_TIMEOUT);

    // ---- release tensor memory -------------------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (comp && warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }

    // ---- partials: [m, l, acc[nacc]] per q-head ------------------------------------------------
    float *ws = a.ws + ((size_t)ul * a.max_splits + split) * G * (2 + D);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const int o = tid + TC_THREADS * w;
        if (o < G * nacc) ws[(o / nacc) * (2 + D) + 2 + o % nacc] = vacc[w];
    }
    if (tid < G) {
        ws[tid * (2 + D)] = sM[tid];
        ws[tid * (2 + D) + 1] = sL[tid];
    }

    // ---- the last split of this kv-head merges all splits ------------------------------------
    __threadfence();
    __syncthreads();
    if (tid == 0) sFlag[0] = (atomicAdd(x.counters + ul, 1) == a.n_split - 1);
    __syncthreads();
    if (!sFlag[0]) return;
    __threadfence();
    float *sBV = reinterpret_cast<float *>(bV);         // B_V rows [D][rV] (bulk copy)
    const bool bv_smem = ok;
    if (bv_smem && tid == 0) {
        mbar_arrive_expect_tx(bar_load, (uint32_t)(D * rV * 4));
        bulk_load(sBV, a.basis[1] + (size_t)ul * D * rV, (uint32_t)(D * rV * 4), bar_load);
    }
    // all q-heads at once: split maxima and sums, per-head weights, then each thread (one channel
    // j) sums its channel over the splits with several independent loads in flight, and the
    // rank-space part is expanded through row j of B_V (read as float4 from L2)
    const int ns = a.n_split, nsc = a.n_split_c;
    const int stride = G * (2 + D);
    const float *wsu = a.ws + (size_t)ul * a.max_splits * stride;
    float *sMw = reinterpret_cast<float *>(bBh);        // [ns][G] maxima, then weights
    float *sLs = sMw + ns * G;                          // [ns][G] sums
    float *sAcc = sP;                                   // [G][D] rank-space sums
    for (int i0 = tid; i0 < ns * G; i0 += 4 * TC_THREADS) {
        float mv[4], lv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * TC_THREADS;
            const float *pw = wsu + (size_t)(i / G) * stride + (i % G) * (2 + D);
            mv[u] = i < ns * G ? __ldcg(pw) : 0.f;
            lv[u] = i < ns * G ? __ldcg(pw + 1) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * TC_THREADS;
            if (i < ns * G) {
                sMw[i] = mv[u];
                sLs[i] = lv[u];
            }
        }
    }
    __syncthreads();
    for (int g = warp; g < G; g += 4) {
        float m = -CUDART_INF_F;
        for (int s2 = lane; s2 < ns; s2 += 32) m = fmaxf(m, sMw[s2 * G + g]);
        m = warp_max_f(m);
        float lsum = 0.f;
        for (int s2 = lane; s2 < ns; s2 += 32) {
            const float w = expf(sMw[s2 * G + g] - m);
            sMw[s2 * G + g] = w;
            lsum = fmaf(w, sLs[s2 * G + g], lsum);
        }
        lsum = warp_sum_f(lsum);
        if (lane == 0) sRed[g] = lsum;
    }
    __syncthreads();
    {
        const int j = tid;
        float accr[GMAX], accw[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) accr[g] = accw[g] = 0.f;
        for (int s0 = 0; s0 < ns; s0 += 16) {
            float v[16][GMAX];
#pragma unroll
            for (int u = 0; u < 16; ++u)
#pragma unroll
                for (int g = 0; g < GMAX; ++g) {
                    const int s2 = s0 + u;
                    v[u][g] = (g < G && s2 < ns && (s2 >= nsc || j < kV))
                                  ? __ldcg(wsu + (size_t)s2 * stride + g * (2 + D) + 2 + j)
                                  : 0.f;
                }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int s2 = s0 + u;
                if (s2 < ns) {
#pragma unroll
                    for (int g = 0; g < GMAX; ++g)
                        if (g < G) {
                            const float w = sMw[s2 * G + g];
                            if (s2 < nsc) accr[g] = fmaf(w, v[u][g], accr[g]);
                            else accw[g] = fmaf(w, v[u][g], accw[g]);
                        }
                }
            }
        }
#pragma unroll
        for (int g = 0; g < GMAX; ++g)
            if (g < G) sAcc[g * D + j] = accr[g];
        __syncthreads();
        float o[GMAX];
#pragma unroll
        for (int g = 0; g < GMAX; ++g) o[g] = accw[g];
        const bool bv_ok = bv_smem && __syncthreads_and(mbar_wait(bar_load, ph_load)) != 0;
        const float *bvrow = bv_ok ? sBV + j * rV : a.basis[1] + ((size_t)ul * D + j) * rV;
        for (int c4 = 0; c4 < kV / 4; ++c4) {
            const float4 b4 = reinterpret_cast<const float4 *>(bvrow)[c4];
#pragma unroll
            for (int g = 0; g < GMAX; ++g)
                if (g < G) {
                    const float *ac = sAcc + g * D + 4 * c4;
                    o[g] = fmaf(ac[0], b4.x, o[g]);
                    o[g] = fmaf(ac[1], b4.y, o[g]);
                    o[g] = fmaf(ac[2], b4.z, o[g]);
                    o[g] = fmaf(ac[3], b4.w, o[g]);
                }
        }
        for (int c = kV & ~3; c < kV; ++c) {
            const float b1 = bvrow[c];
#pragma unroll
            for (int g = 0; g < GMAX; ++g)
                if (g < G) o[g] = fmaf(sAcc[g * D + c], b1, o[g]);
        }
#pragma unroll
        for (int g = 0; g < GMAX; ++g)
            if (g < G) a.out[((size_t)seq * a.H * G + (size_t)h * G + g) * D + j] = o[g] / sRed[g];
    }
    if (tid == 0) x.counters[ul] = 0;
}

cudaError_t launch_decode_tc(const CUtensorMap *tmC, const CUtensorMap *tmB, const DecodeArgs &a,
                             const TcExtra &x, int n_units, cudaStream_t s) {
    const int esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const size_t smem = tc_smem_bytes(x.kblocks, a.r[1], esz);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tc_smem_bytes(2, 128, 4));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    decode_tc_kernel<<<dim3(a.n_split, n_units), TC_THREADS, smem, s>>>(*tmC, *tmB, a, x);
    return cudaGetLastError();
}

}  // namespace iskv
