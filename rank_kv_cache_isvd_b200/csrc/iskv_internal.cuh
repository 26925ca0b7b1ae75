// Internal declarations of the iS-KV CUDA path (kernels + launchers). Not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cuda.h>

#include "iskv.h"

namespace iskv {

constexpr int D = 128;        // head_dim (fixed by the build)
constexpr int DH = D / 2;     // RoPE pairs (j, j + 64)
constexpr int BMAX = 128;     // largest block folded by the in-shared-memory fold kernel
constexpr int BMAX_LARGE = 1024;  // largest block (folded through its triangular factor)
constexpr int LDS = D + 1;    // padded stride of 128-float rows/columns in shared memory
constexpr int GMAX = 8;       // largest GQA group (q-heads per kv-head)
constexpr int DEC_TILE = 128; // decode rows per tile
constexpr int JACOBI_MAX_SWEEPS = 30;

// ---- fold: projection/residual/QR + core SVD + basis update (one CTA per unit and path) ------
struct FoldPath {
    const void *ring;       // [units][R][D] kv dtype
    const float *basis_in;  // [units][D][r]
    float *basis_out;       // [units][D][r]
    const float *sigma_in;  // [units][r] Sigma before the fold (read when k > 0)
    float *sigma_out;       // [units][r] Sigma after the fold
    void *coords;           // [units][n_max][r] fp32, or bf16 when the args' cbf is set
    float *htop;            // [units][r][r]
    int r, k, p, kp;        // rank budget, rank before, residual basis size, rank after
};

struct FoldArgs {
    FoldPath path[2];
    int unit0;              // first unit of the folded set
    long long n_c;          // rows compressed before this fold
    long long n_max;        // coordinate rows per unit
    int slot0;              // ring slot of the oldest exact row (n_c mod R)
    int R;                  // ring capacity (window + block)
    int b;                  // block
    int kv_dtype;
    int *status;
    unsigned long long *stats;  // [0] max sweeps, [1] total sweeps, [2] cores solved
    int skip_new_rows;      // 1: leave the new rows' coordinates to newrows_kernel (large blocks)
    int path_lo, path_hi;   // paths folded: path_lo .. path_hi - 1 (0 = keys, 1 = values)
    int cbf;                // 1: coordinates stored in bf16 (rounded to nearest even)
};

// ---- large blocks (b > BMAX): triangular factor of the block, then the real rows' coordinates -
struct RFactorPath {
    const void *ring;       // [units][R][D] kv dtype
    float *rout;            // [units][128][D] fp32 pseudo-block (R of the block)
    const void *src;        // prefill: rows [call units][src_rows][D] read instead of the ring
    int fbit;               // prefill: rows whose flag has this bit read as zero
};
struct RFactorArgs {
    RFactorPath path[2];
    int unit0, slot0, R, b, kv_dtype;
    int path_lo, path_hi;   // paths processed: path_lo .. path_hi - 1
    long long src_rows;     // prefill: rows per unit of src
    const unsigned char *flags;   // prefill: per-position protection flags [units][flag_stride]
    long long flag_stride;
};
struct NewRowsPath {
    const void *ring;       // [units][R][D] kv dtype
    const float *basis;     // [units][D][r] basis after the fold
    void *coords;           // [units][n_max][r] fp32 or bf16
    int r, kp;
    const void *src;        // prefill: rows [call units][src_rows][D] read instead of the ring
    int fbit;               // prefill: rows whose flag has this bit get zero coordinates
};
struct NewRowsArgs {
    NewRowsPath path[2];
    int unit0, slot0, R, b, kv_dtype;
    long long n_c, n_max;
    int path_lo, path_hi;   // paths processed: path_lo .. path_hi - 1
    int cbf;                // 1: coordinates stored in bf16
    long long src_rows;
    const unsigned char *flags;
    long long flag_stride;
};

// ---- joint per-layer fold (joint_heads): one factorisation over all kv-heads of a (layer, seq) --
// Joint unit j = (layer, sequence) owns kv-head units j H .. j H + H - 1; its basis is stored as
// their per-head slices (d = H D rows in H blocks of D), its coordinates, Sigma and H_top at j.
struct JointPath {
    const void *ring;         // [units][R][D] exact rows per kv-head (kv dtype)
    const float *basis_in;    // [units][D][r] kv-head slices of the joint bases before the fold
    float *basis_out;         // [units][D][r] after the fold
    float *blk;               // [junits][b][D] fp32 pseudo-block F [B P] = [F B | R22^T | 0]
    float *pbasis;            // [junits][D][r] pseudo-basis [I_k; 0]
    const float *pbasis_out;  // [junits][D][r] the fold's basis in the coordinates of [B P]
    float *refl;              // [junits][H][D][ldr] Householder vectors of each kv-head's QR step
    float *tau;               // [junits][H][ldr]
    int r, k, kp;             // rank budget, rank before, rank after
};
struct JointArgs {
    JointPath path[2];
    int junit0;               // first joint unit of the call
    int H;                    // kv-heads per joint unit
    int ldr;                  // column stride of refl (>= k + b of both paths)
    int slot0, R, b, kv_dtype;
    int path_lo, path_hi;     // paths processed: path_lo .. path_hi - 1
};

// ---- prefill protection ------------------------------------------------------------------------
struct ProtArgs {
    const void *keys;       // [call units][src_rows][D] pre-RoPE key rows
    const void *src[2];     // key and value rows, same layout
    long long src_rows;     // rows per unit in the caller's arrays (the prefill length T0)
    long long end;          // rows considered for protection and compression: 0 .. end - 1
    long long T0;
    int chunk, m, suffix, rho;
    int n_chunks, n_chunks_cap;
    float *scores;          // [call units][n_chunks_cap]
    unsigned char *flags;   // [units][flag_stride]: bit 0 key protected, bit 1 value protected
    long long flag_stride;
    int unit0;              // first unit of the call
    int cap;                // protected rows kept per unit and path
    int *ppos[2];           // [units][cap] positions of the protected rows, ascending
    void *store[2];         // [units][cap][D] the protected rows (kv dtype)
    int *pcount[2];         // [units] protected rows stored
    const float2 *rope_cs;  // [max_tokens][DH] (cos, sin) or nullptr (no RoPE)
    int kv_dtype;
    int *status;
};

// ---- history rotation C[0:n] <- C[0:n] H_top (or stale zero-padding) ---------------------------
struct RotPath {
    void *coords;           // [units][n_max][r] fp32 or bf16
    const float *htop;      // [units][r][r]
    int r, k, kp;
};
struct RotArgs {
    RotPath path[2];
    int unit0;
    long long n_old;        // rows to rotate
    long long n_max;
    int stale;              // 1: keep old coordinates (zero columns k..kp-1)
    int path_lo, path_hi;   // paths rotated: path_lo .. path_hi - 1
    int cbf;                // 1: coordinates stored in bf16 (results rounded to nearest even)
};

// ---- window append ----------------------------------------------------------------------------
struct AppendArgs {
    const void *src[2];     // [units][m_total][D] rows of K and V
    void *ring[2];          // [units][R][D]
    int unit0;
    int m_total;            // rows per unit in the caller's array
    int row0;               // first row of this chunk in the caller's array
    int rows;               // rows in this chunk
    long long pos0;         // token position of the chunk's first row
    int R;
    int kv_dtype;
};

// ---- decode -------------------------------------------------------------------------------------
struct DecodeArgs {
    const void *coords[2];  // [units][n_max][r] fp32, or bf16 with cbf (units offset to the layer)
    const float *basis[2];  // [units][D][r]
    const void *ring[2];    // [units][R][D]
    const float2 *rope_cs;  // [max_tokens][DH] (cos, sin) or nullptr
    const float *q;         // [S][QH][D]
    float *out;             // [S][QH][D]
    float *ws;              // [units_in_layer][max_splits][G][2 + D]
    int r[2], k[2];
    long long n_c, t, n_max;
    int R;
    int H, G;               // kv heads, group size
    int split_rows;         // compressed rows per split (multiple of DEC_TILE)
    int n_split_c;          // compressed splits
    int n_split;            // total splits (compressed + window)
    int max_splits;
    int kv_dtype;
    float scale;
    // fused append (tensor-core path only): the row of position new_pos is not yet in the ring;
    // its K and V come from new_row[] ([units][D] kv dtype) and the kernel stores them in the ring
    const void *new_row[2];
    long long new_pos;      // -1: no fused append
    int cbf;                // 1: coordinates stored in bf16 (persistent decode only)
    int cdiv;               // kv-heads sharing one coordinate unit (joint factorisation), else 1
};

// coordinate unit of kv-head unit u (joint factorisation: the kv-heads of a sequence share one)
__host__ __device__ __forceinline__ long long coord_unit(long long u, int cdiv) {
    return cdiv > 1 ? u / cdiv : u;
}

// ---- reconstruct ------------------------------------------------------------------------------
struct ReconArgs {
    const void *coords;     // fp32, or bf16 with cbf
    const float *basis;
    const void *ring;
    const float2 *rope_cs;
    float *out;             // [units][t][D]
    int r, k;
    long long n_c, t, n_max;
    int R, kv_dtype, apply_rope;
    int cbf;
    int cdiv;               // kv-heads sharing one coordinate unit (joint factorisation), else 1
    // prefill protection of this path (pflags nullptr: none); pointers start at the layer's units
    const unsigned char *pflags;
    long long fstride;
    int fbit;               // 1 keys, 2 values
    const int *ppos;        // [units][pcap]
    const void *pstore;     // [units][pcap][D]
    const int *pcount;      // [units]
    int pcap;
};

// extra state of the tensor-core decode kernel
struct TcExtra {
    int kblocks;            // 32-column K-blocks of the key coordinates (ceil(r_K / 32))
    long long row0;         // first coordinate row of this layer in the coordinate tensor map
    int brow0;              // first basis row of this layer (current buffer) in the basis map
    const float4 *rope_t;   // [DH/2][rope_rows] (cos, cos, sin, sin) of pair pairs, or nullptr
    long long rope_rows;
    int *status;
};

// extra state of the warp-specialised persistent decode (decode_ws.cu)
struct WsExtra {
    long long rope_rows;    // rows of the (cos, sin) table a.rope_cs
    long long row0;         // first coordinate row of this layer in the coordinate tensor map
    int brow0;              // first basis row of this layer (current buffer) in the basis map
    int Tc, Tw, Tu;         // tiles per unit: compressed, window; Tu: partition slots per unit
    int W;                  // partition slots of an exact-row (window or protected) tile
    long long N;            // tiles of the layer: units * Tu
    int P;                  // CTAs (one per SM, at most N)
    int maxseg;             // partial records per CTA (units / P + 2)
    int UL;                 // units of the layer
    int factor_bf16;        // 1: coordinates stored in bf16
    int *status;
    // prefill protection (nullptr / 0 when the layer has none); pointers start at the layer's units
    const unsigned char *pflags;  // [units][fstride]: bit 0 key protected, bit 1 value protected
    long long fstride;
    const int *ppos[2];     // [units][pcap] positions of the protected rows, ascending
    const void *pstore[2];  // [units][pcap][D] protected rows (kv dtype)
    const int *pcount[2];   // [units]
    int pcap;
    int Tp;                 // 128-row tiles of protected keys per unit (after the compressed tiles)
};

cudaError_t launch_fold(const FoldArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_rfactor(const RFactorArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_newrows(const NewRowsArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_rotate(const RotArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_joint_prep(const JointArgs &a, int n_junits, cudaStream_t s);
cudaError_t launch_joint_basis(const JointArgs &a, int n_junits, cudaStream_t s);
cudaError_t launch_append(const AppendArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_reconstruct(const ReconArgs &a, int n_units, cudaStream_t s);
cudaError_t launch_coords_to_f32(float *dst, const void *src, size_t n, cudaStream_t s);
cudaError_t launch_protect(const ProtArgs &a, int n_units, cudaStream_t s);
size_t prot_select_smem(int n_chunks, int m);
size_t prot_score_smem(int chunk);
cudaError_t launch_rope_table(float2 *table, long long max_tokens, double theta, cudaStream_t s);
cudaError_t launch_rope_table_t(float4 *table_t, long long max_tokens, double theta,
                                cudaStream_t s);
cudaError_t launch_decode_tc(const CUtensorMap *tmC, const CUtensorMap *tmB, const DecodeArgs &a,
                             const TcExtra &x, int n_units, cudaStream_t s);
cudaError_t launch_decode_ws(const CUtensorMap *tmC, const CUtensorMap *tmB, const DecodeArgs &a,
                             const WsExtra &x, cudaStream_t s);
size_t ws_smem_bytes(int bf, int rV, int esz, int G);
size_t ws_partial_floats(int units, int sms, int G, int rV);
size_t fold_smem_bytes();
size_t tc_smem_bytes(int kblocks, int rV, int esz, int G);

// Stored coordinates: fp32, or bf16 rounded to nearest even from the fp32 result.
__device__ __forceinline__ float load_coord(const void *base, size_t idx, int cbf) {
    if (cbf) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
    return reinterpret_cast<const float *>(base)[idx];
}
__device__ __forceinline__ void store_coord(void *base, size_t idx, float v, int cbf) {
    if (cbf)
        reinterpret_cast<__nv_bfloat16 *>(base)[idx] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float *>(base)[idx] = v;
}

__device__ __forceinline__ float load_row_elem(const void *base, size_t idx, int kv_dtype) {
    if (kv_dtype == ISKV_BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
    return reinterpret_cast<const float *>(base)[idx];
}

// Raises `fn`'s dynamic shared-memory limit on the current device to at least `bytes`. Function
// attributes belong to a device, so the largest value set so far is remembered per device in
// `done` (64 entries, zero-initialised by the caller).
inline cudaError_t ensure_smem(const void *fn, size_t bytes, size_t *done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (bytes <= done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done[dev] = bytes;
    return e;
}

__device__ __forceinline__ void set_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace iskv
