// Decode attention over the compressed cache, warp-specialised and persistent (sm_100a: TMA,
// tcgen05 tensor cores with TMEM accumulators, mbarrier pipelines).
//
// iS-KV summary, "Reconstruction and Storage": compressed row i is (C B^T)[i] (C = U Sigma), the
// window rows are exact. Keys are compressed before RoPE, so a tile of 128 reconstructed keys
// K~ = C_K[tile] B_K^T is formed on the tensor cores (three-term tf32 for fp32 factors) and rotated
// afterwards. RoPE at position t0 + tau (tile start t0, row tau) is split into two rotations:
//   score_g = sum_j Re( conj(Q_gj e^{-i w_j t0}) * (k_j e^{i w_j tau}) ),  k_j = K~_j + i K~_{j+64},
// so the queries are rotated once per tile (by t0) and every row by an angle that depends only on
// tau. The cosines and sines of row tau are written once into the row's tensor-memory lane and
// read back next to the row's key values (no per-row global table reads). Values are accumulated in rank space (sum_i p_i C_V[i]) and expanded once through
// B_V^T by the merge kernel.
//
// Work split: the (unit, tile) pairs of all units of the layer - each unit's compressed tiles
// followed by its window tiles - are cut into one contiguous range per CTA (one CTA per SM), so
// every SM streams the same number of tiles. A CTA's range covers segments of one or more units;
// each segment leaves one partial (running max, sum, rank-space and channel-space accumulators)
// per q-head, and the merge kernel combines the partials of a unit with log-sum-exp weights.
//
// Warp roles (12 warps):
//   warp 0      TMA producer: queries, B_K, key-coordinate tiles (K ring), value tiles (V ring);
//   warps 1-3   split the fp32 key tiles into tf32 hi + lo parts; warp 1 issues the MMAs into one
//               of two TMEM accumulators and commits them to the ring barriers;
//   warps 4-11  epilogue: two threads per row (TMEM lane = row, each half of the RoPE pairs);
//               rotation and dot products, online softmax, value sums, partial records.
// Every wait is bounded: a wait that gives up raises a CTA-wide abort flag, the sticky device
// status is set to ISKV_ERR_TIMEOUT, and the CTA drains its own copies and MMAs before it exits.
#include <math_constants.h>

#include "iskv_internal.cuh"
#include "tc_util.cuh"

namespace iskv {

constexpr int WS_THREADS = 384;
constexpr int WS_EPI = 256;                  // epilogue threads (warps 4 .. 11)
constexpr int WS_NSK = 2;                    // key-coordinate stages
constexpr int WS_MAXSV = 4;                  // value stages (at most)
constexpr uint32_t WS_BLK = 128u * 128u;     // 128 rows x 128 bytes
constexpr int BAR_EPI = 1, BAR_SPLIT = 3, BAR_ALL = 4;   // named barriers (groups: 1 and 2)
constexpr float LOG2E = 1.4426950408889634f;
// Lazy softmax reference: probabilities are 2^(s - m_ref) with m_ref a CTA-uniform running
// reference that moves only when a score exceeds it by more than WS_LAZY (log2 units), so that
// p <= 2^WS_LAZY and sums over a unit stay far inside the fp32 range.
constexpr float WS_LAZY = 20.f;
// register split: producer/split warpgroup, epilogue warpgroups, and the per-thread count the
// launch must grant for it (128 x 64 + 256 x 200 = 384 x 154.7)
constexpr int WS_REG_LO = 64, WS_REG_HI = 200, WS_REG_LAUNCH = 160;
static_assert(128 * WS_REG_LO + 256 * WS_REG_HI <= WS_THREADS * WS_REG_LAUNCH,
              "register split exceeds the launch allocation");

struct WsLayout {
    uint32_t bh, bl, kst, vst, q, eg, smax, ssum, sfl, sidx, cs, bars, total;
    uint32_t kstage, vstage;
    int nsv;
};

// Shared-memory plan. fp32 coordinates: a K stage holds the tile's tf32 hi part (in place) and its
// lo part; bf16 coordinates: the tile only (exact bf16 operands). Each epilogue group owns an area
// of q~ [2][G][128] and p [2][128][G] floats (its segment-end reduction aliases it).
__host__ __device__ inline WsLayout ws_layout(int bf, int rV, int esz, int G, uint32_t limit) {
    WsLayout L;
    uint32_t o = 0;
    // B_K terms: fp32 coordinates use tf32 (hi, lo); bf16 coordinates use three bf16 terms of the
    // fp32 basis (hi, mid, lo: 24 significant bits), the third at bl + WS_BLK
    L.bh = o; o += WS_BLK;
    L.bl = o; o += bf ? 2u * WS_BLK : WS_BLK;
    L.kstage = bf ? WS_BLK : 2u * WS_BLK;
    L.kst = o; o += WS_NSK * L.kstage;
    const uint32_t vc = 128u * rV * (bf ? 2u : 4u), vw = 128u * D * esz;
    L.vstage = ((vc > vw ? vc : vw) + 1023u) & ~1023u;
    L.vst = o;
    const uint32_t misc = (uint32_t)G * 512u * 2u            // q, two segment slots
                          + (uint32_t)G * 4096u              // the two groups' areas
                          + 64u * 4u + 32u * 4u              // smax, ssum
                          + 2u * 2u * 128u * 5u              // per-row flags and store indices
                          + 2u * (uint32_t)G * DH * 8u       // next tiles' (cos, sin) of the queries
                          + 512u + 1024u;                    // barriers, alignment slack
    int nsv = WS_MAXSV;
    while (nsv > 2 && o + nsv * L.vstage + misc > limit) --nsv;
    L.nsv = nsv;
    o += nsv * L.vstage;
    L.q = o; o += G * 512u * 2u;
    L.eg = o; o += G * 4096u;
    L.smax = o; o += 64u * 4u;
    L.ssum = o; o += 32u * 4u;
    L.sfl = o; o += 2u * 2u * 128u;                         // protection flags of the tiles' rows
    L.sidx = o; o += 2u * 2u * 128u * 4u;                   // their value-store indices
    L.cs = o; o += 2u * (uint32_t)G * DH * 8u;              // (cos, sin) for the groups' next q~
    L.bars = o; o += 512u;
    L.total = o + 1024u;
    return L;
}

size_t ws_smem_bytes(int bf, int rV, int esz, int G) {
    return ws_layout(bf, rV, esz, G, 227u * 1024u).total;
}

// ---- small device helpers --------------------------------------------------------------------
__device__ __forceinline__ bool mbar_try(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// try_wait that may suspend the thread for up to `ns` nanoseconds while the phase is incomplete
// (the thread resumes as soon as it completes), so that waiting warps issue almost nothing.
__device__ __forceinline__ bool mbar_try_for(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return done != 0;
}

// Polls of a suspending wait before it gives up: each poll suspends for at most WS_SUSPEND_NS, and
// 2^18 polls of even a microsecond are far longer than any launch.
constexpr uint32_t WS_POLL_LIMIT = 1u << 18, WS_SUSPEND_NS = 20000;

// Bounded wait that also gives up as soon as another role raised the abort flag.
__device__ __forceinline__ bool wait_ab(uint64_t *bar, uint32_t parity, volatile int *abort,
                                        bool = false) {
    for (uint32_t i = 0; i < WS_POLL_LIMIT; ++i) {
        if (mbar_try_for(bar, parity, WS_SUSPEND_NS)) return true;
        if (*abort) return false;
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void bar_named(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Named barrier that also returns the AND of `v` over the participating threads.
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Named barrier that also returns the OR of `v` over the participating threads.
__device__ __forceinline__ bool bar_or(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void ws_griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void ws_griddep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Tensor-memory columns: two key accumulators of 128 columns, then the per-row RoPE table (cos of
// the 64 pairs, then their sin), 384 of the 512 allocated.
constexpr uint32_t WS_TMEM_COLS = 512, WS_TAB = 256;

// 8 consecutive fp32 columns of this thread's TMEM lane <- v (visible after tmem_wait_st).
__device__ __forceinline__ void tmem_st8x(uint32_t taddr, const float (&v)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One 16-lane x 8-column block of tensor memory in the 16x256b fragment: thread t holds (lane
// t/4, columns 2(t%4) and 2(t%4)+1) in v[0], v[1] and (lane t/4 + 8, the same columns) in v[2],
// v[3]; taddr addresses the block's first lane and column.
__device__ __forceinline__ void tmem_ld4f(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st4f(uint32_t taddr, const float (&v)[4]) {
    asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3]))
                 : "memory");
}

// The key-phase operands of one 8-pair group for the thread's four rows (16x256b fragments):
// [block][4]: cos lanes 0-15, sin lanes 0-15, key real, key imaginary, then the same at lanes 16-31.
struct KeyBlk {
    float v[8][4];
};

// Loads of one 8-pair group [j0, j0 + 8): the RoPE table and the key accumulator, both lane halves.
__device__ __forceinline__ void key_blk_load(KeyBlk &kb, uint32_t tab, uint32_t acc, uint32_t ln0,
                                             uint32_t ln16, int j0) {
#pragma unroll
    for (int lh = 0; lh < 2; ++lh) {
        const uint32_t ln = lh ? ln16 : ln0;
        tmem_ld4f(tab + ln + j0, kb.v[4 * lh + 0]);
        tmem_ld4f(tab + ln + DH + j0, kb.v[4 * lh + 1]);
        tmem_ld4f(acc + ln + j0, kb.v[4 * lh + 2]);
        tmem_ld4f(acc + ln + DH + j0, kb.v[4 * lh + 3]);
    }
}

// Waits for this thread's tensor-memory loads; the loaded registers pass through the wait, so no
// use of them can be scheduled before it.
__device__ __forceinline__ void key_blk_wait(KeyBlk &kb) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(kb.v[0][0]), "+f"(kb.v[0][1]), "+f"(kb.v[0][2]), "+f"(kb.v[0][3]),
                   "+f"(kb.v[1][0]), "+f"(kb.v[1][1]), "+f"(kb.v[1][2]), "+f"(kb.v[1][3]),
                   "+f"(kb.v[2][0]), "+f"(kb.v[2][1]), "+f"(kb.v[2][2]), "+f"(kb.v[2][3]),
                   "+f"(kb.v[3][0]), "+f"(kb.v[3][1]), "+f"(kb.v[3][2]), "+f"(kb.v[3][3]),
                   "+f"(kb.v[4][0]), "+f"(kb.v[4][1]), "+f"(kb.v[4][2]), "+f"(kb.v[4][3]),
                   "+f"(kb.v[5][0]), "+f"(kb.v[5][1]), "+f"(kb.v[5][2]), "+f"(kb.v[5][3]),
                   "+f"(kb.v[6][0]), "+f"(kb.v[6][1]), "+f"(kb.v[6][2]), "+f"(kb.v[6][3]),
                   "+f"(kb.v[7][0]), "+f"(kb.v[7][1]), "+f"(kb.v[7][2]), "+f"(kb.v[7][3])
                 :
                 : "memory");
}

// 8-byte asynchronous copy global -> shared (this thread waits for its own copies).
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 8 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld8x(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 with bf16 operands, one CTA.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// fp32 values in place -> their tf32 "hi" part (top 19 bits); the exact remainder "lo" at the
// same offset of `lo`. Threads t0 .. t0 + nt - 1 of the CTA share the work.
__device__ __forceinline__ void split_tf32_range(uint8_t *hi, uint8_t *lo, int bytes, int t,
                                                 int nt) {
    float4 *h4 = reinterpret_cast<float4 *>(hi);
    float4 *l4 = reinterpret_cast<float4 *>(lo);
    for (int i = t; i < bytes / 16; i += nt) {
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

// Three bf16 terms (hi + mid + lo, 24 significant bits) of a fp32 basis [D][rK] (rK <= 64, even),
// written as 128 rows x 64 columns (zero beyond rK) in the 128-byte-swizzled K-major layout: the
// 16-byte chunk c of row n sits at chunk c ^ (n mod 8). Threads t, t + nt, ... share the work.
__device__ __forceinline__ void build_b_terms(uint8_t *bh, uint8_t *bm, uint8_t *bl,
                                              const float *B, int rK, int t, int nt) {
    for (int p = t; p < 128 * 32; p += nt) {
        const int n = p >> 5, k = (p & 31) * 2;
        float v0 = 0.f, v1 = 0.f;
        if (k < rK) {
            const float2 f = *reinterpret_cast<const float2 *>(B + (size_t)n * rK + k);
            v0 = f.x;
            v1 = f.y;
        }
        const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
        const float r0 = v0 - __low2float(h), r1 = v1 - __high2float(h);
        const __nv_bfloat162 m = __floats2bfloat162_rn(r0, r1);
        const __nv_bfloat162 l = __floats2bfloat162_rn(r0 - __low2float(m), r1 - __high2float(m));
        const uint32_t byte = (uint32_t)k * 2u;
        const uint32_t off = (uint32_t)n * 128u + ((((byte >> 4) ^ (uint32_t)(n & 7)) << 4) | (byte & 15u));
        *reinterpret_cast<__nv_bfloat162 *>(bh + off) = h;
        *reinterpret_cast<__nv_bfloat162 *>(bm + off) = m;
        *reinterpret_cast<__nv_bfloat162 *>(bl + off) = l;
    }
}

// 8 consecutive channels of an exact row (bf16 or fp32) as fp32.
__device__ __forceinline__ void load_row8(const void *base, size_t idx, int kv_dtype,
                                          float (&v)[8]) {
    if (kv_dtype == ISKV_BF16) {
        const uint4 u = *reinterpret_cast<const uint4 *>(
            reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + idx);
        const float4 a = p[0], b = p[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// 4 consecutive channels (idx a multiple of 4) of an exact row (bf16 or fp32) as fp32.
__device__ __forceinline__ float4 load_row4(const void *base, size_t idx, int kv_dtype) {
    if (kv_dtype == ISKV_BF16) {
        const uint2 u = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(base) + idx);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    return *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + idx);
}

// Index of `key` in the ascending array a[0 .. n), or -1.
__device__ __forceinline__ int find_sorted(const int *a, int n, int key) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] < key) lo = mid + 1;
        else hi = mid;
    }
    return (lo < n && a[lo] == key) ? lo : -1;
}

// The G probabilities of one row (vector loads: rows are 4 G bytes apart, 16-byte aligned for G = 4).
template <int GT>
__device__ __forceinline__ void load_p(const float *p, float (&v)[GT]) {
    if constexpr (GT == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        v[0] = x.x;
        v[1] = x.y;
        v[2] = x.z;
        v[3] = x.w;
    } else if constexpr (GT == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x;
        v[1] = x.y;
    } else {
#pragma unroll
        for (int g = 0; g < GT; ++g) v[g] = p[g];
    }
}

// The G probabilities of one row, stored (the row's G floats are 4 G bytes apart: 16-byte aligned
// for G = 4).
template <int GT>
__device__ __forceinline__ void store_p(float *p, const float (&v)[GT]) {
    if constexpr (GT == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (GT == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int g = 0; g < GT; ++g) p[g] = v[g];
    }
}

// Four consecutive values of a staged value row: fmt 2 = bf16, 4 = fp32.
__device__ __forceinline__ float4 load_v4s(const uint8_t *row, int c, int fmt) {
    if (fmt == 2) {
        const uint2 u = *reinterpret_cast<const uint2 *>(row + 2 * c);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    return *reinterpret_cast<const float4 *>(row + 4 * c);
}

// The CTA's tile range and the segment (unit, first tile, end tile) containing tile g.
struct WsRange {
    long long g0, g1;
};
// First tile of a unit whose partition slot is at or after slot o: the Tc compressed tiles take
// one slot each, every exact-row tile (protected or window) W slots.
__host__ __device__ inline int ws_vtile(int o, int Tc, int W) {
    return o <= Tc ? o : Tc + (o - Tc + W - 1) / W;
}

__device__ __forceinline__ WsRange ws_range(const WsExtra &x, int c) {
    WsRange r;
    r.g0 = (long long)c * x.N / x.P;
    r.g1 = (long long)(c + 1) * x.N / x.P;
    return r;
}

// ---- the split kernel --------------------------------------------------------------------------
template <bool BF, int GT>
__global__ void __launch_bounds__(WS_THREADS, 1) decode_ws_kernel(
    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmB,
    DecodeArgs a, WsExtra x) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int G = GT;
    const int rV = a.r[1];
    const int esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const WsLayout L = ws_layout(BF ? 1 : 0, rV, esz, G, 227u * 1024u);
    const int NSV = L.nsv;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *k_full = bars, *k_empty = bars + 2, *v_full = bars + 4, *v_empty = bars + 8;
    uint64_t *b_full = bars + 12, *b_empty = bars + 13, *acc_full = bars + 14,
             *acc_empty = bars + 16, *q_full = bars + 18, *q_empty = bars + 20;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 22);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 23);
    int *counters = reinterpret_cast<int *>(bars + 24);    // [8] progress, read at teardown
    float *sQ = reinterpret_cast<float *>(sm + L.q);        // [2 slots][G][128]
    float *sMax = reinterpret_cast<float *>(sm + L.smax);   // [2 groups][2][4][4]
    float *sSum = reinterpret_cast<float *>(sm + L.ssum);   // [2 groups][4 warps][4] probability sums
    unsigned char *sFl = sm + L.sfl;                        // [2 groups][2][128] row flags
    int *sIdx = reinterpret_cast<int *>(sm + L.sidx);       // [2 groups][2][128] value-store indices
    float2 *sCs = reinterpret_cast<float2 *>(sm + L.cs);    // [2 groups][G * 64] (cos, sin)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const WsRange rg = ws_range(x, blockIdx.x);
    const int Tc = x.Tc, Tu = x.Tu;
    const long long u_first = rg.g0 / Tu;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(k_full + i, 1);
            mbar_init(k_empty + i, 1);
            mbar_init(acc_full + i, 1);
            mbar_init(acc_empty + i, 4);
            mbar_init(q_full + i, 1);
            mbar_init(q_empty + i, 8);
        }
        for (int i = 0; i < WS_MAXSV; ++i) {
            mbar_init(v_full + i, 1);
            mbar_init(v_empty + i, 4);
        }
        mbar_init(b_full, 1);
        mbar_init(b_empty, 1);
        *abort_flag = 0;
        for (int i = 0; i < 8; ++i) counters[i] = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, WS_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // registers move from the producer/split warpgroup to the two epilogue warpgroups; the launch
    // grants at least WS_REG_LAUNCH per thread (checked on the host before the first launch), so
    // 128 x WS_REG_LO + 256 x WS_REG_HI fits the block's allocation
    if (warp < 4)
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(WS_REG_LO));
    else
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(WS_REG_HI));

    // every segment of this CTA, in order: unit u, tiles [ta, tb) of the unit (those whose first
    // partition slot lies in the CTA's range; possibly none), and the slots it spans
    auto seg_of = [&](long long g, long long &u, int &ta, int &tb, int &adv) {
        u = g / Tu;
        const int o0 = (int)(g - u * Tu);
        const int o1 = (int)min((long long)Tu, o0 + (rg.g1 - g));
        ta = ws_vtile(o0, Tc, x.W);
        tb = ws_vtile(o1, Tc, x.W);
        adv = o1 - o0;
    };

    if (warp == 0) {
        // ==================================== producer ===========================================
        int kt = 0, vt = 0, seg = 0, bseg = 0;
        int vs = 0;                                     // V stage of tile vt, and its pass parity
        uint32_t vph = 0;
        ws_griddep_wait();
        if (lane == 0) {
            bool ok = true;
            for (long long g = rg.g0; g < rg.g1 && ok;) {
                long long u;
                int ta, tb, adv;
                seg_of(g, u, ta, tb, adv);
                const int seq = (int)(u / a.H), h = (int)(u % a.H);
                // queries of this unit's q-heads
                const int qs = seg & 1;
                ok = wait_ab(q_empty + qs, ((seg >> 1) & 1) ^ 1, abort_flag, true);
                if (!ok) break;
                mbar_arrive_expect_tx(q_full + qs, (uint32_t)(G * D * 4));
                bulk_load(sQ + qs * G * D, a.q + ((size_t)seq * a.H * G + (size_t)h * G) * D,
                          (uint32_t)(G * D * 4), q_full + qs);
                ++seg;
                counters[0] = seg;
                if (!BF && ta < Tc) {
                    // B_K of this unit (one buffer; free once the previous segment's MMAs are done)
                    ok = wait_ab(b_empty, (bseg & 1) ^ 1, abort_flag, true);
                    if (!ok) break;
                    mbar_arrive_expect_tx(b_full, WS_BLK);
                    tma_load_2d(sm + L.bh, &tmB, 0, x.brow0 + (int)u * D, b_full);
                    ++bseg;
                    counters[1] = bseg;
                }
                for (int tl = ta; tl < tb && ok; ++tl) {
                    const bool comp = tl < Tc;
                    if (!comp && tl < Tc + x.Tp) continue;     // protected rows: read by the epilogue
                    long long t0;
                    int rows;
                    if (comp) {
                        t0 = (long long)tl * DEC_TILE;
                        rows = (int)min((long long)DEC_TILE, a.n_c - t0);
                        const int ks = kt % WS_NSK;
                        ok = wait_ab(k_empty + ks, ((kt / WS_NSK) & 1) ^ 1, abort_flag, true);
                        if (!ok) break;
                        mbar_arrive_expect_tx(k_full + ks, WS_BLK);
                        tma_load_2d(sm + L.kst + ks * L.kstage, &tmC, 0,
                                    (int)(x.row0 + coord_unit(u, a.cdiv) * a.n_max + t0), k_full + ks);
                        ++kt;
                        counters[2] = kt;
                    } else {
                        t0 = a.n_c + (long long)(tl - Tc - x.Tp) * DEC_TILE;
                        rows = (int)min((long long)DEC_TILE, a.t - t0);
                    }
                    ok = wait_ab(v_empty + vs, vph ^ 1, abort_flag, true);
                    if (!ok) break;
                    uint8_t *dst = sm + L.vst + vs * L.vstage;
                    if (comp) {
                        const uint32_t fsz = BF ? 2u : 4u;
                        const uint32_t nb = (uint32_t)rows * rV * fsz;
                        mbar_arrive_expect_tx(v_full + vs, nb);
                        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.coords[1]) +
                                             ((size_t)coord_unit(u, a.cdiv) * a.n_max + t0) * rV * fsz;
                        bulk_load(dst, src, nb, v_full + vs);
                    } else {
                        const int s0 = (int)(t0 % a.R);
                        const int n1 = min(rows, a.R - s0);
                        const uint32_t rb = D * esz;
                        const char *ring = static_cast<const char *>(a.ring[1]) +
                                           (size_t)u * a.R * D * esz;
                        mbar_arrive_expect_tx(v_full + vs, (uint32_t)rows * rb);
                        bulk_load(dst, ring + (size_t)s0 * rb, (uint32_t)n1 * rb, v_full + vs);
                        if (n1 < rows)
                            bulk_load(dst + (size_t)n1 * rb, ring, (uint32_t)(rows - n1) * rb,
                                      v_full + vs);
                    }
                    ++vt;
                    if (++vs == NSV) {
                        vs = 0;
                        vph ^= 1;
                    }
                    counters[3] = vt;
                }
                g += adv;
            }
        }
    } else if (warp < 4) {
        // =============================== split + MMA issue =======================================
        const int st = tid - 32;                        // 0 .. 95
        int kt = 0, at = 0, bseg = 0;
        ws_griddep_wait();
        bool ok = true;
        const uint32_t idesc = BF ? idesc_bf16(128, 128) : idesc_tf32(128, 128);
        for (long long g = rg.g0; g < rg.g1 && ok;) {
            long long u;
            int ta, tb, adv;
            seg_of(g, u, ta, tb, adv);
            g += adv;
            if (ta >= Tc) continue;
            bool w;
            if (BF) {
                // three bf16 terms of this unit's fp32 basis, written in the 128-byte-swizzled
                // K-major layout, once the previous segment's MMAs no longer read them
                w = wait_ab(b_empty, (bseg & 1) ^ 1, abort_flag, true);
                if (w) {
                    build_b_terms(sm + L.bh, sm + L.bl, sm + L.bl + WS_BLK,
                                  a.basis[0] + (size_t)u * D * a.r[0], a.r[0], st, 96);
                    fence_proxy_async_smem();
                }
            } else {
                w = wait_ab(b_full, bseg & 1, abort_flag, true);
                if (w) {
                    split_tf32_range(sm + L.bh, sm + L.bl, WS_BLK, st, 96);
                    fence_proxy_async_smem();
                }
            }
            ok = bar_and(BAR_SPLIT, 96, w);
            if (!ok) break;
            ++bseg;
            const int te = min(tb, Tc);
            for (int tl = ta; tl < te; ++tl) {
                const int ks = kt % WS_NSK;
                uint8_t *A = sm + L.kst + ks * L.kstage;
                w = wait_ab(k_full + ks, (kt / WS_NSK) & 1, abort_flag, true);
                if (!BF && w) {
                    split_tf32_range(A, A + WS_BLK, WS_BLK, st, 96);
                    fence_proxy_async_smem();
                }
                ok = bar_and(BAR_SPLIT, 96, w);
                if (!ok) break;
                if (st == 0) {
                    const int buf = at & 1;
                    bool e = wait_ab(acc_empty + buf, ((at >> 1) & 1) ^ 1, abort_flag, true);
                    if (e) {
                        tc_fence_after();
                        const uint32_t d = tmem + 128u * buf;
                        const uint32_t aH = smem_u32(A), bH = smem_u32(sm + L.bh);
                        if (BF) {
                            // C (exact bf16) times the three terms of B; K steps of 16 columns
                            const int nk = (a.r[0] + 15) >> 4;
                            const uint32_t bM = smem_u32(sm + L.bl), bL = bM + WS_BLK;
                            for (int kk = 0; kk < nk; ++kk) {
                                const uint32_t off = kk * 32;
                                mma_bf16(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bH + off),
                                         idesc, kk > 0);
                                mma_bf16(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bM + off),
                                         idesc, 1);
                                mma_bf16(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bL + off),
                                         idesc, 1);
                            }
                        } else {
                            const uint32_t aL = aH + WS_BLK, bL = smem_u32(sm + L.bl);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t off = kk * 32;
                                mma_tf32(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bH + off),
                                         idesc, kk > 0);
                                mma_tf32(d, sw128_kmajor_desc(aH + off), sw128_kmajor_desc(bL + off),
                                         idesc, 1);
                                mma_tf32(d, sw128_kmajor_desc(aL + off), sw128_kmajor_desc(bH + off),
                                         idesc, 1);
                            }
                        }
                        mma_commit(acc_full + buf);
                        mma_commit(k_empty + ks);
                        if (tl + 1 == te) mma_commit(b_empty);
                        counters[4] = at + 1;
                        counters[5] = kt + 1;
                    }
                    // on a failed wait the abort flag is raised: every thread's next wait gives up
                    // and the next split barrier ends the loop for the whole group
                }
                __syncwarp();
                ++kt;
                ++at;
            }
        }
    } else {
        // ==================================== epilogue ===========================================
        // Two groups of four warps (one warp per tensor-memory lane quarter) take alternate tiles of
        // the CTA's range, so that one group's key phase (FMA pipe) overlaps the other's softmax and
        // value sums. Key phase: warp qw covers rows 32 qw .. 32 qw + 31 and all 64 RoPE pairs;
        // thread t = (r0, q4) handles rows 32 qw + r0 + 8 m (m = 0 .. 3) and, in every 8-pair group
        // [j0, j0 + 8), the pairs j0 + 2 q4 and j0 + 2 q4 + 1 (the 16x256b fragment), so each query
        // value read from shared memory serves four rows; a quad reduction leaves thread t with the
        // full score of row tau = 32 qw + r0 + 8 q4 for every q-head.
        const int et = tid - 128;                       // 0 .. 255
        const int ew = warp - 4, qw = warp & 3, gid = ew >> 2;
        const int gt = et & 127;                        // thread within the group
        const int bar_g = BAR_EPI + gid;                // the group's named barrier
        const int q4 = lane & 3, r0 = lane >> 2;
        const int tau = 32 * qw + r0 + 8 * q4;
        const uint32_t lane0 = (uint32_t)(qw * 32) << 16, lane16 = (uint32_t)(qw * 32 + 16) << 16;
        // row m's rotation e^{i w_j tau_m} for the thread's pairs, fixed for the kernel, kept in
        // tensor memory next to the key accumulators (cos at WS_TAB + j, sin at WS_TAB + 64 + j):
        // group g writes the rows of lane half g (16-byte loads, all issued before the stores)
        {
            const int lh = gid;
            float4 t[8][2];
#pragma unroll
            for (int k = 0; k < 8; ++k)
#pragma unroll
                for (int rs = 0; rs < 2; ++rs) {
                    const int row = 32 * qw + 16 * lh + r0 + 8 * rs;
                    t[k][rs] = make_float4(1.f, 0.f, 1.f, 0.f);
                    if (a.rope_cs != nullptr && row < x.rope_rows)
                        t[k][rs] = *reinterpret_cast<const float4 *>(a.rope_cs + (size_t)row * DH + 8 * k + 2 * q4);
                }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float cv[4] = {t[k][0].x, t[k][0].z, t[k][1].x, t[k][1].z};
                const float sv[4] = {t[k][0].y, t[k][0].w, t[k][1].y, t[k][1].w};
                const uint32_t tl0 = tmem + WS_TAB + (lh ? lane16 : lane0) + 8 * k;
                tmem_st4f(tl0, cv);
                tmem_st4f(tl0 + DH, sv);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        bar_named(BAR_ALL, WS_EPI);
        tc_fence_after();
        ws_griddep_wait();
        const float qscale = a.scale * LOG2E;           // scores in log2 units
        // group areas: q~ [2][G][128], p [2][128][G]; the segment-end reduction aliases them
        float *sQt = reinterpret_cast<float *>(sm + L.eg) + (size_t)gid * 4 * G * 128;
        float *sP = sQt + 2 * G * 128;
        float4 *sRed = reinterpret_cast<float4 *>(sQt);          // [4 warps][G][32]
        float *sMaxg = sMax + gid * 32, *sSumg = sSum + gid * 16;
        unsigned char *sFlg = sFl + gid * 256;
        int *sIdxg = sIdx + gid * 256;
        float2 *sCsg = sCs + gid * G * DH;
        // value-sum layout of the group: thread = (quad qd, slice sl); compressed tiles use kV's
        // quads, exact rows the 32 channel quads
        const int nqr = (rV + 3) >> 2;
        const int nqpr = nqr <= 8 ? 8 : nqr <= 16 ? 16 : 32;
        const int qdr = gt & (nqpr - 1), slr = gt / nqpr, nslr = 128 / nqpr;
        const int qdw = gt & 31, slw = gt >> 5;
        bool ok = true;
        int at = 0, vt = 0, seg = 0, it = 0, own = 0;
        int vs = 0;                                     // V stage of tile vt, and its pass parity
        uint32_t vph = 0;

        // start position of tile tl of a unit: compressed, protected (queries unrotated: each
        // protected row carries its own angle), window
        auto tile_t0 = [&](int tl) -> long long {
            if (tl < Tc) return (long long)tl * DEC_TILE;
            if (tl < Tc + x.Tp) return 0;
            return a.n_c + (long long)(tl - Tc - x.Tp) * DEC_TILE;
        };
        // q~ = (q rotated by -w_j t0) * scale * log2(e) for tile start t0, into the group's q~ buffer
        // b; thread gt builds pairs gt and gt + 128 of the G x 64 pairs
        auto make_qt = [&](const float *q, long long t0, int b, bool from_cs) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = gt + 128 * h;
                if (e < G * DH) {
                    const int g = e / DH, j = e & (DH - 1);
                    float2 cs = make_float2(1.f, 0.f);
                    if (a.rope_cs != nullptr) cs = from_cs ? sCsg[e] : a.rope_cs[(size_t)t0 * DH + j];
                    const float qr = q[g * D + j], qi = q[g * D + DH + j];
                    sQt[(b * G + g) * D + j] = qscale * fmaf(qr, cs.x, qi * cs.y);
                    sQt[(b * G + g) * D + DH + j] = qscale * fmaf(qi, cs.x, -qr * cs.y);
                }
            }
        };

        for (long long g = rg.g0; g < rg.g1 && ok;) {
            long long u;
            int ta, tb, adv;
            seg_of(g, u, ta, tb, adv);
            g += adv;
            const int jseg = (int)(u - u_first);
            const int qs = seg & 1;
            bool w = wait_ab(q_full + qs, (seg >> 1) & 1, abort_flag);
            const float *q = sQ + qs * G * D;
            // m_ref (uniform over the group), this thread's probability sums and the value sums,
            // all relative to 2^m_ref
            float mref[GT], lth[GT];
            float4 vr[GT], vw[GT];
#pragma unroll
            for (int gg = 0; gg < GT; ++gg) {
                mref[gg] = -CUDART_INF_F;
                lth[gg] = 0.f;
                vr[gg] = make_float4(0.f, 0.f, 0.f, 0.f);
                vw[gg] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            // this group's first tile of the segment
            const int tf = ta + ((it & 1) != gid ? 1 : 0);
            if (w && tf < tb) make_qt(q, tile_t0(tf), own & 1, false);
            ok = bar_and(bar_g, 128, w);
            if (!ok) break;
            bool good = true;                       // this thread's waits of the segment so far
            // channel-space sums: window or protected tiles, or value-protected compressed rows
            const bool has_c = ta < Tc, has_w = tb > Tc || (x.pflags != nullptr && ta < Tc);
            const int npk = x.pflags != nullptr ? x.pcount[0][u] : 0;
            const int npv = x.pflags != nullptr ? x.pcount[1][u] : 0;
            for (int tl = ta; tl < tb; ++tl) {
                const bool comp = tl < Tc;
                const bool prot = !comp && tl < Tc + x.Tp;       // protected exact keys
                if ((it & 1) != gid) {
                    // the other group's tile: keep the ring and accumulator counters in step
                    if (comp) ++at;
                    if (!prot) {
                        ++vt;
                        if (++vs == NSV) {
                            vs = 0;
                            vph ^= 1;
                        }
                    }
                    ++it;
                    continue;
                }
                const int b = own & 1;
                const long long t0 = tile_t0(tl);
                // this group's next tile of the segment (two ahead): its query rotation, copied now
                const bool nxt = tl + 2 < tb;
                if (nxt && a.rope_cs != nullptr) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int e = gt + 128 * h;
                        if (e < G * DH)
                            cp_async8(sCsg + e, a.rope_cs + (size_t)tile_t0(tl + 2) * DH + (e & (DH - 1)));
                    }
                }
                int rows;
                long long pos;
                unsigned char fl = 0;
                int vidx = -1;
                if (prot) {
                    const int pi = (tl - Tc) * DEC_TILE;
                    rows = max(0, min(DEC_TILE, npk - pi));
                    pos = tau < rows ? x.ppos[0][(size_t)u * x.pcap + pi + tau] : 0;
                    if (tau < rows) vidx = find_sorted(x.ppos[1] + (size_t)u * x.pcap, npv, (int)pos);
                } else {
                    rows = (int)min((long long)DEC_TILE, (comp ? a.n_c : a.t) - t0);
                    pos = t0 + tau;
                    if (comp && x.pflags != nullptr && tau < rows) {
                        fl = x.pflags[(size_t)u * x.fstride + pos];
                        if ((fl & 2) && !(fl & 1))
                            vidx = find_sorted(x.ppos[1] + (size_t)u * x.pcap, npv, (int)pos);
                    }
                }
                // rows whose key is protected are attended in the protected tiles
                const bool valid = tau < rows && !(fl & 1);
                // ---- key phase: partial scores of the thread's four rows (float2: two pairs) ------
                float2 acc[4][GT];
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int gg = 0; gg < GT; ++gg) acc[m][gg] = make_float2(0.f, 0.f);
                bool wk = true;
                if (comp) wk = wait_ab(acc_full + (at & 1), (at >> 1) & 1, abort_flag);
                // the tensor-memory loads below are warp-collective: decide per warp
                wk = __all_sync(0xffffffffu, wk);
                good = good && wk;
                tc_fence_after();
                const float *qt = sQt + b * G * D;
                int xrows = 0;
                if (!comp) {
                    const int pi = prot ? (tl - Tc) * DEC_TILE : 0;
                    xrows = prot ? max(0, min(DEC_TILE, npk - pi)) : (int)min((long long)DEC_TILE, a.t - t0);
                }
                const uint32_t acc0 = tmem + 128u * (at & 1);
                // rotate row m's key of the pair group [j0, j0 + 8) and dot it with the queries
                auto key_math = [&](int j0, const float2 (&kr2)[4], const float2 (&ki2)[4],
                                    const float2 (&cc2)[4], const float2 (&ss2)[4]) {
                    float2 qre[GT], qim[GT];
#pragma unroll
                    for (int gg = 0; gg < GT; ++gg) {
                        qre[gg] = *reinterpret_cast<const float2 *>(qt + gg * D + j0 + 2 * q4);
                        qim[gg] = *reinterpret_cast<const float2 *>(qt + gg * D + DH + j0 + 2 * q4);
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 k1 = kr2[m], k2 = ki2[m], c2 = cc2[m], s2 = ss2[m];
                        const float2 t1 = __fmul2_rn(k2, s2);
                        const float2 zr = __ffma2_rn(k1, c2, make_float2(-t1.x, -t1.y));
                        const float2 zi = __ffma2_rn(k1, s2, __fmul2_rn(k2, c2));
#pragma unroll
                        for (int gg = 0; gg < GT; ++gg) {
                            acc[m][gg] = __ffma2_rn(qre[gg], zr, acc[m][gg]);
                            acc[m][gg] = __ffma2_rn(qim[gg], zi, acc[m][gg]);
                        }
                    }
                };
                auto key_math_blk = [&](int j0, const KeyBlk &kb) {
                    float2 kr2[4], ki2[4], cc2[4], ss2[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int lh = m >> 1, o = 2 * (m & 1);
                        cc2[m] = make_float2(kb.v[4 * lh + 0][o], kb.v[4 * lh + 0][o + 1]);
                        ss2[m] = make_float2(kb.v[4 * lh + 1][o], kb.v[4 * lh + 1][o + 1]);
                        kr2[m] = wk ? make_float2(kb.v[4 * lh + 2][o], kb.v[4 * lh + 2][o + 1]) : make_float2(0.f, 0.f);
                        ki2[m] = wk ? make_float2(kb.v[4 * lh + 3][o], kb.v[4 * lh + 3][o + 1]) : make_float2(0.f, 0.f);
                    }
                    key_math(j0, kr2, ki2, cc2, ss2);
                };
                if (comp) {
                    // tensor-memory loads of the next pair group in flight while this one computes
                    KeyBlk ka, kb;
                    key_blk_load(ka, tmem + WS_TAB, acc0, lane0, lane16, 0);
                    key_blk_wait(ka);
#pragma unroll 1
                    for (int k = 0; k < 8; k += 2) {
                        key_blk_load(kb, tmem + WS_TAB, acc0, lane0, lane16, 8 * (k + 1));
                        key_math_blk(8 * k, ka);
                        key_blk_wait(kb);
                        if (k + 2 < 8) key_blk_load(ka, tmem + WS_TAB, acc0, lane0, lane16, 8 * (k + 2));
                        key_math_blk(8 * (k + 1), kb);
                        if (k + 2 < 8) key_blk_wait(ka);
                    }
                } else {
#pragma unroll 1
                    for (int k = 0; k < 8; ++k) {
                        const int j0 = 8 * k;
                        // rows from the exact stores; protected rows rotate by their full position
                        // (their queries are unrotated), window rows by their offset in the tile
                        float2 kr2[4], ki2[4], cc2[4], ss2[4];
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const int row = 32 * qw + r0 + 8 * m;
                            float kr[2] = {0.f, 0.f}, ki[2] = {0.f, 0.f}, cc[2] = {1.f, 1.f}, ss[2] = {0.f, 0.f};
                            if (row < xrows) {
                                const void *src;
                                size_t base;
                                long long apos;
                                if (prot) {
                                    const size_t pidx = (size_t)u * x.pcap + (tl - Tc) * DEC_TILE + row;
                                    src = x.pstore[0];
                                    base = pidx * D;
                                    apos = x.ppos[0][pidx];
                                } else {
                                    const long long p = t0 + row;
                                    const bool fresh = p == a.new_pos;
                                    src = fresh ? a.new_row[0] : a.ring[0];
                                    base = fresh ? (size_t)u * D
                                                 : ((size_t)u * a.R + (unsigned)p % (unsigned)a.R) * D;
                                    apos = row;
                                }
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int j = j0 + 2 * q4 + e;
                                    kr[e] = load_row_elem(src, base + j, a.kv_dtype);
                                    ki[e] = load_row_elem(src, base + DH + j, a.kv_dtype);
                                    if (a.rope_cs != nullptr) {
                                        const float2 c = a.rope_cs[(size_t)apos * DH + j];
                                        cc[e] = c.x;
                                        ss[e] = c.y;
                                    }
                                }
                            }
                            kr2[m] = make_float2(kr[0], kr[1]);
                            ki2[m] = make_float2(ki[0], ki[1]);
                            cc2[m] = make_float2(cc[0], cc[1]);
                            ss2[m] = make_float2(ss[0], ss[1]);
                        }
                        key_math(j0, kr2, ki2, cc2, ss2);
                    }
                }
                if (comp) {
                    // the accumulator is read: let the MMA warp reuse it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0 && wk) mbar_arrive(acc_empty + (at & 1));
                    ++at;
                }
                // quad reduction: thread q4 ends with row m = q4 (tile row tau), all 64 pairs
                float sc[GT];
                {
                    float s1[2][GT];
                    const bool hi2 = (q4 & 2) != 0;
#pragma unroll
                    for (int i = 0; i < 2; ++i)
#pragma unroll
                        for (int gg = 0; gg < GT; ++gg) {
                            const float lo_s = acc[i][gg].x + acc[i][gg].y;
                            const float hi_s = acc[2 + i][gg].x + acc[2 + i][gg].y;
                            const float keep = hi2 ? hi_s : lo_s, send = hi2 ? lo_s : hi_s;
                            s1[i][gg] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                        }
                    const bool odd = (q4 & 1) != 0;
#pragma unroll
                    for (int gg = 0; gg < GT; ++gg) {
                        const float keep = odd ? s1[1][gg] : s1[0][gg], send = odd ? s1[0][gg] : s1[1][gg];
                        const float full = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                        sc[gg] = valid ? full : -CUDART_INF_F;
                    }
                }
                // ---- the group's next tile's queries; probabilities against m_ref ------------------
                if (nxt) {
                    if (a.rope_cs != nullptr) cp_async_wait_all();
                    make_qt(q, 0, b ^ 1, true);
                }
                sFlg[b * 128 + tau] = (unsigned char)((fl & 2) && !(fl & 1) && vidx >= 0 ? 2 : 0);
                sIdxg[b * 128 + tau] = vidx;
                float pv[GT];
                bool over = false;
#pragma unroll
                for (int gg = 0; gg < GT; ++gg) {
                    const float dlt = sc[gg] - mref[gg];          // +inf or NaN while m_ref is unset
                    over = over || (valid && !(dlt <= WS_LAZY));
                    pv[gg] = valid ? ex2(dlt) : 0.f;
                }
                store_p<GT>(sP + (b * 128 + tau) * G, pv);
                if (bar_or(bar_g, 128, over)) {
                    // some score is above m_ref + WS_LAZY (or m_ref is unset): m_ref <- the running
                    // maximum, rescale the sums, recompute this tile's probabilities
#pragma unroll
                    for (int gg = 0; gg < GT; ++gg) {
                        float m = sc[gg];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane == 0) sMaxg[(b * 4 + qw) * 4 + gg] = m;
                    }
                    bar_named(bar_g, 128);
#pragma unroll
                    for (int gg = 0; gg < GT; ++gg) {
                        const float mt = fmaxf(fmaxf(sMaxg[(b * 4 + 0) * 4 + gg], sMaxg[(b * 4 + 1) * 4 + gg]),
                                               fmaxf(sMaxg[(b * 4 + 2) * 4 + gg], sMaxg[(b * 4 + 3) * 4 + gg]));
                        const float mn = fmaxf(mref[gg], mt);
                        // a tile without rows leaves the running state as it is
                        const float alpha = mn == -CUDART_INF_F ? 1.f : ex2(mref[gg] - mn);
                        mref[gg] = mn;
                        lth[gg] *= alpha;
                        const float2 al = make_float2(alpha, alpha);
                        float2 x01 = __fmul2_rn(al, make_float2(vr[gg].x, vr[gg].y));
                        float2 x23 = __fmul2_rn(al, make_float2(vr[gg].z, vr[gg].w));
                        vr[gg] = make_float4(x01.x, x01.y, x23.x, x23.y);
                        x01 = __fmul2_rn(al, make_float2(vw[gg].x, vw[gg].y));
                        x23 = __fmul2_rn(al, make_float2(vw[gg].z, vw[gg].w));
                        vw[gg] = make_float4(x01.x, x01.y, x23.x, x23.y);
                        pv[gg] = valid ? ex2(sc[gg] - mn) : 0.f;
                    }
                    store_p<GT>(sP + (b * 128 + tau) * G, pv);
                    bar_named(bar_g, 128);
                }
#pragma unroll
                for (int gg = 0; gg < GT; ++gg) lth[gg] += pv[gg];
                // ---- value sums: v_g += sum_i p[g][i] V[i][quad] ----------------------------
                const bool wv = prot ? true : wait_ab(v_full + vs, vph, abort_flag);
                good = good && wv;
                const uint8_t *V = sm + L.vst + vs * L.vstage;
                const float *P = sP + (size_t)b * 128 * G;
                if (prot) {
                    // protected rows: exact values from the value store (channel sums)
                    for (int i = slw; i < rows; i += 4) {
                        const int vi = sIdxg[b * 128 + i];
                        if (vi < 0) continue;
                        const float4 v4 = load_row4(x.pstore[1], ((size_t)u * x.pcap + vi) * D + 4 * qdw, a.kv_dtype);
                        const float2 v01 = make_float2(v4.x, v4.y), v23 = make_float2(v4.z, v4.w);
                        float pp[GT];
                        load_p(P + i * G, pp);
#pragma unroll
                        for (int gg = 0; gg < GT; ++gg) {
                            const float2 p2 = make_float2(pp[gg], pp[gg]);
                            const float2 x01 = __ffma2_rn(p2, v01, make_float2(vw[gg].x, vw[gg].y));
                            const float2 x23 = __ffma2_rn(p2, v23, make_float2(vw[gg].z, vw[gg].w));
                            vw[gg] = make_float4(x01.x, x01.y, x23.x, x23.y);
                        }
                    }
                } else if (wv) {
                    if (comp && x.pflags != nullptr) {
                        // value-protected rows of a compressed tile: their coordinates are zero;
                        // the exact value row enters the channel sums
                        for (int i = slw; i < rows; i += 4) {
                            if (!(sFlg[b * 128 + i] & 2)) continue;
                            const int vi = sIdxg[b * 128 + i];
                            const float4 v4 = load_row4(x.pstore[1], ((size_t)u * x.pcap + vi) * D + 4 * qdw, a.kv_dtype);
                            const float2 v01 = make_float2(v4.x, v4.y), v23 = make_float2(v4.z, v4.w);
                            float pp[GT];
                            load_p(P + i * G, pp);
#pragma unroll
                            for (int gg = 0; gg < GT; ++gg) {
                                const float2 p2 = make_float2(pp[gg], pp[gg]);
                                const float2 x01 = __ffma2_rn(p2, v01, make_float2(vw[gg].x, vw[gg].y));
                                const float2 x23 = __ffma2_rn(p2, v23, make_float2(vw[gg].z, vw[gg].w));
                                vw[gg] = make_float4(x01.x, x01.y, x23.x, x23.y);
                            }
                        }
                    }
                    if (comp) {
                        const int vld = rV * (BF ? 2 : 4);
#pragma unroll 4
                        for (int i = slr; i < rows; i += nslr) {
                            const float4 v = load_v4s(V + (size_t)i * vld, 4 * qdr, BF ? 2 : 4);
                            const float2 v01 = make_float2(v.x, v.y), v23 = make_float2(v.z, v.w);
                            float pp[GT];
                            load_p(P + i * G, pp);
#pragma unroll
                            for (int gg = 0; gg < GT; ++gg) {
                                const float pg = pp[gg];
                                const float2 p2 = make_float2(pg, pg);
                                const float2 x01 = __ffma2_rn(p2, v01, make_float2(vr[gg].x, vr[gg].y));
                                const float2 x23 = __ffma2_rn(p2, v23, make_float2(vr[gg].z, vr[gg].w));
                                vr[gg] = make_float4(x01.x, x01.y, x23.x, x23.y);
                            }
                        }
                    } else {
                        const int vld = D * esz;
                        const int inew = (a.new_pos >= t0 && a.new_pos < t0 + rows)
                                             ? (int)(a.new_pos - t0) : -1;
#pragma unroll 4
                        for (int i = slw; i < rows; i += 4) {
                            float4 v;
                            if (i == inew) {
                                v = load_row4(a.new_row[1], (size_t)u * D + 4 * qdw, a.kv_dtype);
                            } else {
                                v = load_v4s(V + (size_t)i * vld, 4 * qdw, esz);
                            }
                            const float2 v01 = make_float2(v.x, v.y), v23 = make_float2(v.z, v.w);
                            float pp[GT];
                            load_p(P + i * G, pp);
#pragma unroll
                            for (int gg = 0; gg < GT; ++gg) {
                                const float pg = pp[gg];
                                const float2 p2 = make_float2(pg, pg);
                                const float2 x01 = __ffma2_rn(p2, v01, make_float2(vw[gg].x, vw[gg].y));
                                const float2 x23 = __ffma2_rn(p2, v23, make_float2(vw[gg].z, vw[gg].w));
                                vw[gg] = make_float4(x01.x, x01.y, x23.x, x23.y);
                            }
                        }
                        if (inew >= 0 && gt < D) {
                            // fused append: store the new position's K and V rows in the ring
                            const size_t slot = ((size_t)u * a.R + (size_t)(a.new_pos % a.R)) * D + gt;
                            if (a.kv_dtype == ISKV_BF16) {
                                const __nv_bfloat16 *nk = static_cast<const __nv_bfloat16 *>(a.new_row[0]) + (size_t)u * D;
                                const __nv_bfloat16 *nv = static_cast<const __nv_bfloat16 *>(a.new_row[1]) + (size_t)u * D;
                                const_cast<__nv_bfloat16 *>(static_cast<const __nv_bfloat16 *>(a.ring[0]))[slot] = nk[gt];
                                const_cast<__nv_bfloat16 *>(static_cast<const __nv_bfloat16 *>(a.ring[1]))[slot] = nv[gt];
                            } else {
                                const float *nk = static_cast<const float *>(a.new_row[0]) + (size_t)u * D;
                                const float *nv = static_cast<const float *>(a.new_row[1]) + (size_t)u * D;
                                const_cast<float *>(static_cast<const float *>(a.ring[0]))[slot] = nk[gt];
                                const_cast<float *>(static_cast<const float *>(a.ring[1]))[slot] = nv[gt];
                            }
                        }
                    }
                }
                __syncwarp();
                if (!prot) {
                    if (lane == 0) mbar_arrive(v_empty + vs);
                    ++vt;
                    if (++vs == NSV) {
                        vs = 0;
                        vph ^= 1;
                    }
                }
                ++own;
                ++it;
            }
            // q slot consumed (every q~ of the segment is built)
            __syncwarp();
            if (lane == 0) mbar_arrive(q_empty + qs);
            ++seg;
            ok = bar_and(bar_g, 128, ok && good);         // tiles done: the reduction area is free
            if (!ok) break;
            // ---- this group's partial record: [m, l, acc_rank[rV], acc_chan[D]] per q-head ----------
            float *rec = a.ws + (((size_t)blockIdx.x * x.maxseg + jseg) * 2 + gid) * G * (2 + rV + D);
            const int gw = ew & 3;                          // warp within the group
            if (has_c) {
#pragma unroll
                for (int gg = 0; gg < GT; ++gg) {
                    for (int o = nqpr; o < 32; o <<= 1) {
                        vr[gg].x += __shfl_xor_sync(0xffffffffu, vr[gg].x, o);
                        vr[gg].y += __shfl_xor_sync(0xffffffffu, vr[gg].y, o);
                        vr[gg].z += __shfl_xor_sync(0xffffffffu, vr[gg].z, o);
                        vr[gg].w += __shfl_xor_sync(0xffffffffu, vr[gg].w, o);
                    }
                    if (lane < nqpr) sRed[(gw * G + gg) * 32 + qdr] = vr[gg];
                }
                bar_named(bar_g, 128);
                for (int o = gt; o < G * rV; o += 128) {
                    const int gg = o / rV, c = o % rV;
                    float s = 0.f;
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4)
                        s += reinterpret_cast<const float *>(sRed)[((w4 * G + gg) * 32) * 4 + c];
                    rec[gg * (2 + rV + D) + 2 + c] = s;
                }
                bar_named(bar_g, 128);
            } else {
                for (int o = gt; o < G * rV; o += 128)
                    rec[(o / rV) * (2 + rV + D) + 2 + o % rV] = 0.f;
            }
            if (has_w) {
#pragma unroll
                for (int gg = 0; gg < GT; ++gg) sRed[(gw * G + gg) * 32 + qdw] = vw[gg];
                bar_named(bar_g, 128);
                for (int o = gt; o < G * D; o += 128) {
                    const int gg = o / D, c = o % D;
                    float s = 0.f;
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4)
                        s += reinterpret_cast<const float *>(sRed)[((w4 * G + gg) * 32) * 4 + c];
                    rec[gg * (2 + rV + D) + 2 + rV + c] = s;
                }
                bar_named(bar_g, 128);
            } else {
                for (int o = gt; o < G * D; o += 128)
                    rec[(o / D) * (2 + rV + D) + 2 + rV + o % D] = 0.f;
            }
            // probability sums: per warp, then over the group's 4 warps
#pragma unroll
            for (int gg = 0; gg < GT; ++gg) {
                float sl = lth[gg];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, o);
                if (lane == 0) sSumg[gw * 4 + gg] = sl;
            }
            bar_named(bar_g, 128);
            if (gt < G) {
#pragma unroll
                for (int gg = 0; gg < GT; ++gg)
                    if (gg == gt) {
                        float l = 0.f;
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4) l += sSumg[w4 * 4 + gg];
                        rec[gg * (2 + rV + D)] = mref[gg];
                        rec[gg * (2 + rV + D) + 1] = l;
                    }
            }
            // the next segment rewrites the group area (aliased by the reduction)
            bar_named(bar_g, 128);
        }
        if (et == 0) {
            counters[6] = at;
            counters[7] = vt;
        }
    }

    // ---- teardown: after an abort, wait (bounded) for this CTA's own copies and MMAs ------------
    ws_griddep_launch();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        set_status(x.status, ISKV_ERR_TIMEOUT);
        // loads issued but never consumed, and MMAs committed but never read
        const int kt_p = counters[2], kt_m = counters[5];
        for (int n = kt_m; n < kt_p; ++n) mbar_wait(k_full + n % WS_NSK, (n / WS_NSK) & 1);
        const int at_m = counters[4], at_e = counters[6];
        for (int n = at_e; n < at_m; ++n) mbar_wait(acc_full + (n & 1), (n >> 1) & 1);
        if (at_m > 0) mbar_wait(acc_full + ((at_m - 1) & 1), ((at_m - 1) >> 1) & 1);
        const int vt_p = counters[3], vt_e = counters[7];
        for (int n = vt_e; n < vt_p; ++n) mbar_wait(v_full + n % NSV, (n / NSV) & 1);
        const int q_p = counters[0];
        if (q_p > 0) mbar_wait(q_full + ((q_p - 1) & 1), ((q_p - 1) >> 1) & 1);
        const int b_p = counters[1];
        if (b_p > 0) mbar_wait(b_full, (b_p - 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, WS_TMEM_COLS);
    }
}

// ---- merge: one CTA of 256 threads per (unit, q-head) ----------------------------------------------
// The unit's records (two per CTA whose range touches it) are read in parallel: first the q-head's
// references and sums, then every output element's weighted sum over the records, with the loads
// of all records independent; the rank-space sum is expanded once through B_V^T.
constexpr int WM_THREADS = 256;

__host__ __device__ inline int ws_merge_records(int P) { return 2 * P; }

template <int GT>
__global__ void __launch_bounds__(WM_THREADS) decode_ws_merge_kernel(DecodeArgs a, WsExtra x) {
    extern __shared__ float msm[];
    const int G = GT, rV = a.r[1], kV = a.k[1];
    const int ldb = kV | 1;
    const int RM = ws_merge_records(x.P);
    float *sBV = msm;                                   // [D][ldb]
    float *sAcc = sBV + D * ldb;                        // [rV] rank-space sums
    float *sCh = sAcc + rV;                             // [D] channel-space sums
    float *sW = sCh + D;                                // [RM] record references, then weights
    float *sL = sW + RM;                                // [RM] record sums
    float *sML = sL + RM;                               // [2]: reference M, sum L
    unsigned long long *sOff = reinterpret_cast<unsigned long long *>(sML + 2);   // [RM]
    const int u = blockIdx.x, g = blockIdx.y;
    const int seq = u / a.H, h = u % a.H;
    const int tid = threadIdx.x;
    ws_griddep_launch();
    if (kV > 0) {
        const float *B = a.basis[1] + (size_t)u * D * rV;
        for (int o = tid; o < D * kV; o += WM_THREADS) sBV[(o / kV) * ldb + o % kV] = B[(size_t)(o / kV) * rV + o % kV];
    }
    ws_griddep_wait();
    // CTAs whose tile ranges touch this unit, and the unit's segment index in each
    const long long x0 = (long long)u * x.Tu, x1 = (long long)(u + 1) * x.Tu - 1;
    const int c_lo = (int)(((x0 + 1) * x.P + x.N - 1) / x.N) - 1;
    const int c_hi = (int)(((x1 + 1) * x.P + x.N - 1) / x.N) - 1;
    const int R = 2 * (c_hi - c_lo + 1);
    const int rs = 2 + rV + D;                          // floats per q-head in a record
    // record r: CTA c_lo + r / 2, group r % 2, at the unit's segment index in that CTA; this
    // q-head's part of it
    for (int r = tid; r < R; r += WM_THREADS) {
        const int c = c_lo + (r >> 1);
        const long long g0 = (long long)c * x.N / x.P;
        const int js = (int)(u - g0 / x.Tu);
        const unsigned long long off =
            (((unsigned long long)c * x.maxseg + js) * 2 + (r & 1)) * (unsigned long long)G * rs +
            (unsigned long long)g * rs;
        sOff[r] = off;
        sW[r] = __ldcg(a.ws + off);
        sL[r] = __ldcg(a.ws + off + 1);
    }
    __syncthreads();
    if (tid < 32) {
        // reference (warp max) and weights; a group that saw no tile of the unit left m = -inf
        float m = -CUDART_INF_F;
        for (int r = tid; r < R; r += 32) m = fmaxf(m, sW[r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int r = tid; r < R; r += 32) {
            const float mr = sW[r];
            const float w = mr == -CUDART_INF_F ? 0.f : ex2(mr - m);
            sW[r] = w;
            l = fmaf(w, sL[r], l);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (tid == 0) {
            sML[0] = m;
            sML[1] = l;
        }
    }
    __syncthreads();
    // weighted sums of the rank-space (c < rV) and channel-space (c >= rV) parts
    for (int c = tid; c < rV + D; c += WM_THREADS) {
        float acc = 0.f;
#pragma unroll 4
        for (int r = 0; r < R; ++r) acc = fmaf(sW[r], __ldcg(a.ws + sOff[r] + 2 + c), acc);
        if (c < rV) sAcc[c] = acc;
        else sCh[c - rV] = acc;
    }
    __syncthreads();
    for (int j = tid; j < D; j += WM_THREADS) {
        const float *br = sBV + j * ldb;
        float v = sCh[j];
        for (int c = 0; c < kV; ++c) v = fmaf(sAcc[c], br[c], v);
        a.out[((size_t)seq * a.H * G + (size_t)h * G + g) * D + j] = v / sML[1];
    }
}

size_t ws_merge_smem_bytes(int kV, int rV, int G, int P) {
    (void)G;
    // floats (an even count: the 8-byte record offsets follow aligned), then the offsets
    return ((size_t)D * (kV | 1) + (size_t)rV + (size_t)D + 2 * (size_t)ws_merge_records(P) + 2 + 1) /
               2 * 2 * sizeof(float) +
           (size_t)ws_merge_records(P) * 8 + 8;
}

size_t ws_partial_floats(int units, int sms, int G, int rV) {
    return ((size_t)units + 2 * (size_t)sms) * 2 * G * (2 + rV + D);
}

// The register split inside the kernel waits for registers that the launch must have granted:
// refuse to launch a build whose register count is below WS_REG_LAUNCH.
template <bool BF, int GT>
static bool ws_regs_ok() {
    static int ok = -1;
    if (ok < 0) {
        cudaFuncAttributes fa;
        ok = (cudaFuncGetAttributes(&fa, decode_ws_kernel<BF, GT>) == cudaSuccess &&
              ((fa.numRegs + 7) & ~7) >= WS_REG_LAUNCH)
                 ? 1
                 : 0;
        if (!ok) cudaGetLastError();
    }
    return ok == 1;
}

template <bool BF, int GT>
static cudaError_t launch_ws_t(const CUtensorMap *tmC, const CUtensorMap *tmB, const DecodeArgs &a,
                               const WsExtra &x, cudaStream_t s, size_t smem, size_t msmem) {
    static size_t attr[64] = {0}, mattr[64] = {0};
    if (!ws_regs_ok<BF, GT>()) return cudaErrorInvalidConfiguration;
    cudaError_t e = ensure_smem((const void *)decode_ws_kernel<BF, GT>, smem, attr);
    if (e != cudaSuccess) return e;
    e = ensure_smem((const void *)decode_ws_merge_kernel<GT>, msmem, mattr);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr1[1];
    attr1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr1[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(x.P);
    cfg.blockDim = dim3(WS_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr1;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_ws_kernel<BF, GT>, *tmC, *tmB, a, x);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(x.UL, GT);
    cfg.blockDim = dim3(WM_THREADS);
    cfg.dynamicSmemBytes = msmem;
    return cudaLaunchKernelEx(&cfg, decode_ws_merge_kernel<GT>, a, x);
}

cudaError_t launch_decode_ws(const CUtensorMap *tmC, const CUtensorMap *tmB, const DecodeArgs &a,
                             const WsExtra &x, cudaStream_t s) {
    const int esz = a.kv_dtype == ISKV_BF16 ? 2 : 4;
    const size_t smem = ws_smem_bytes(x.factor_bf16, a.r[1], esz, a.G);
    const size_t msmem = ws_merge_smem_bytes(a.k[1], a.r[1], a.G, x.P);
    const bool bf = x.factor_bf16 != 0;
    switch (a.G) {
    case 1: return bf ? launch_ws_t<true, 1>(tmC, tmB, a, x, s, smem, msmem)
                      : launch_ws_t<false, 1>(tmC, tmB, a, x, s, smem, msmem);
    case 2: return bf ? launch_ws_t<true, 2>(tmC, tmB, a, x, s, smem, msmem)
                      : launch_ws_t<false, 2>(tmC, tmB, a, x, s, smem, msmem);
    case 4: return bf ? launch_ws_t<true, 4>(tmC, tmB, a, x, s, smem, msmem)
                      : launch_ws_t<false, 4>(tmC, tmB, a, x, s, smem, msmem);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace iskv
