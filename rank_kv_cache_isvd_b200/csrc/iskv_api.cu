// Host side of the C ABI declared in include/iskv.h: configuration checks, device allocation,
// per-layer counters (tokens t, compressed rows n_c, current ranks, basis buffer), the fold
// schedule and launch sequencing. No device work happens outside the kernels in this directory.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <new>
#include <vector>

#include "iskv_internal.cuh"

using namespace iskv;

struct iskv_handle {
    iskv_config cfg;
    int device = 0;
    int sms = 148;
    int U = 0;            // units per path: n_layers * batch * n_kv_heads
    int UL = 0;           // units per layer
    int R = 0;            // ring rows per unit
    int G = 1;
    int NB = 2;           // buffers of basis / Sigma / H_top per path (ring indexed by fold number)
    long long n_max = 0;  // coordinate rows per unit
    int max_splits = 0;
    size_t esz = 2;
    void *coords[2] = {nullptr, nullptr};  // fp32, or bf16 with coord_bf16
    int cbf = 0;                          // coordinates stored in bf16
    size_t csz = 4;                       // bytes per stored coordinate
    float *basis[2] = {nullptr, nullptr};   // [NB][U][D][r]
    float *sigma[2] = {nullptr, nullptr};   // [NB][U][r]
    float *htop[2] = {nullptr, nullptr};    // [NB][U][r][r]
    float *rbig[2] = {nullptr, nullptr};    // [U][128][D] triangular factor of a large block
    // joint per-layer factorisation (joint_heads): joint unit j = layer * batch + seq holds the
    // coordinates, Sigma and H_top of all kv-heads of that (layer, sequence); its basis is stored
    // as the kv-heads' slices at units j H + h
    bool joint = false;
    int JL = 0;           // joint units per layer (batch)
    int CU = 0;           // coordinate units per path: U, or n_layers * batch when joint
    int CL = 0;           // coordinate units per layer: UL, or batch when joint
    int ldr = 0;          // column stride of jrefl: max over paths of rank + block
    float *jblk[2] = {nullptr, nullptr};    // [CU][b][D] pseudo-blocks
    float *jpb[2] = {nullptr, nullptr};     // [CU][D][r] pseudo-bases [I_k; 0]
    float *jpbo[2] = {nullptr, nullptr};    // [CU][D][r] fold results in pseudo coordinates
    float *jrefl[2] = {nullptr, nullptr};   // [CU][n_kv][D][ldr] Householder vectors per kv-head
    float *jtau[2] = {nullptr, nullptr};    // [CU][n_kv][ldr]
    void *ring[2] = {nullptr, nullptr};
    float2 *rope_cs = nullptr;
    float4 *rope_t = nullptr;             // transposed copy for the tensor-core decode
    float *ws = nullptr;
    int *status = nullptr;
    unsigned long long *stats = nullptr;  // fold statistics (3 counters)
    bool tc = false;                      // tensor-core decode available for this shape
    bool ws_ok = false;                   // warp-specialised persistent decode for this shape
    CUtensorMap tmC;                      // key coordinates [U * n_max][r_K], 32 x 128 boxes
    CUtensorMap tmB;                      // key bases [NB * U * D][r_K]
    // per layer
    std::vector<long long> t, nc;
    std::vector<int> kcur[2];             // ranks as of the last applied fold (what decode reads)
    std::vector<long long> nf;            // folds launched
    std::vector<long long> pbase;         // rows compressed by the layer's prefill (0: none)
    std::vector<int> pfold;               // 1 if the layer's prefill counts as its first update
    std::vector<int> ptiles;              // 128-row tiles of the largest protected key store
    std::vector<unsigned char> pact;      // the layer's prefill protected some positions
    // prefill protection (prot_cap > 0): per-position flags, protected stores, counts, scores
    int pcap = 0;
    unsigned char *pflags = nullptr;      // [U][n_max]: bit 0 key protected, bit 1 value protected
    int *ppos[2] = {nullptr, nullptr};    // [U][pcap] positions, ascending
    void *pstore[2] = {nullptr, nullptr}; // [U][pcap][D] rows (kv dtype)
    int *pcount[2] = {nullptr, nullptr};  // [U]
    float *pscores = nullptr;             // [UL][n_max] chunk scores of one layer
    std::vector<int> kf[2];               // ranks after the last launched fold
    std::vector<int> fk;                  // [layer][NB][4]: k_K, kp_K, k_V, kp_V of fold j % NB
    std::vector<unsigned char> on_side;   // [layer][NB]: fold j % NB ran on an internal stream
    // look-ahead folding: internal streams and completion events
    static constexpr int NS = 4;
    cudaStream_t side[NS] = {nullptr, nullptr, nullptr, nullptr};
    std::vector<cudaEvent_t> done;        // [layer][NB]
    cudaEvent_t fork = nullptr;
    long long launches = 0;
};

namespace {

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int now = -1;
        if (prev >= 0 && cudaGetDevice(&now) == cudaSuccess && now != prev) cudaSetDevice(prev);
    }
};

int rank_of(const iskv_handle *h, int which) { return which ? h->cfg.rank_v : h->cfg.rank_k; }

long long ncomp(long long t, int block, int window) {
    const long long x = t - window;
    return x > 0 ? (long long)block * (x / block) : 0;
}

void free_all(iskv_handle *h) {
    for (int x = 0; x < 2; ++x) {
        cudaFree(h->coords[x]);
        cudaFree(h->basis[x]);
        cudaFree(h->sigma[x]);
        cudaFree(h->ring[x]);
        cudaFree(h->htop[x]);
        cudaFree(h->rbig[x]);
        cudaFree(h->jblk[x]);
        cudaFree(h->jpb[x]);
        cudaFree(h->jpbo[x]);
        cudaFree(h->jrefl[x]);
        cudaFree(h->jtau[x]);
    }
    cudaFree(h->rope_cs);
    cudaFree(h->rope_t);
    cudaFree(h->pflags);
    cudaFree(h->pscores);
    for (int x = 0; x < 2; ++x) {
        cudaFree(h->ppos[x]);
        cudaFree(h->pstore[x]);
        cudaFree(h->pcount[x]);
    }
    cudaFree(h->ws);
    cudaFree(h->status);
    cudaFree(h->stats);
    for (cudaEvent_t e : h->done)
        if (e) cudaEventDestroy(e);
    if (h->fork) cudaEventDestroy(h->fork);
    for (int i = 0; i < iskv_handle::NS; ++i)
        if (h->side[i]) cudaStreamDestroy(h->side[i]);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D tensor [rows][cols] (row stride cols) of fp32 or bf16 elements, boxes of 128 bytes (32 fp32
// or 64 bf16 columns; columns past `cols` read as zero) x 128 rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int cols, long long rows, bool bf16 = false) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn || rows < 1 || rows > 0x7fffffffLL) return false;
    const size_t esz = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool valid_layer(const iskv_handle *h, int layer) {
    return layer >= 0 && layer < h->cfg.n_layers;
}

float *basis_buf(const iskv_handle *h, int x, int i) {
    return h->basis[x] + (size_t)i * h->U * D * rank_of(h, x);
}
float *sigma_buf(const iskv_handle *h, int x, int i) {
    return h->sigma[x] + (size_t)i * h->U * rank_of(h, x);
}
float *htop_buf(const iskv_handle *h, int x, int i) {
    const size_t r = (size_t)rank_of(h, x);
    return h->htop[x] + (size_t)i * h->U * r * r;
}
// Fixed-basis mode: fold j of path x only stores the block's coordinates in the frozen basis once
// the first ceil(min(r, d) / b) folds (which fill the rank budget) have run.
bool frozen(const iskv_handle *h, int x, long long j) {
    if (!h->cfg.fixed_basis) return false;
    const int r = rank_of(h, x) < D ? rank_of(h, x) : D;
    return j >= (r + h->cfg.block - 1) / h->cfg.block;
}

// Fold index of a layer holding nc compressed positions, and the first position of fold j's block.
// Without a prefill the folds take blocks 0, b, 2b, ...; after a prefill of pbase rows (which
// counts as update 0) fold j takes the block at pbase + (j - 1) b.
long long fold_of(const iskv_handle *h, int layer, long long nc) {
    return h->pfold[layer] + (nc - h->pbase[layer]) / h->cfg.block;
}
long long block_start(const iskv_handle *h, int layer, long long j) {
    return h->pbase[layer] + (j - h->pfold[layer]) * (long long)h->cfg.block;
}

// buffer of the basis / Sigma produced by the last applied fold
int current_buffer(const iskv_handle *h, int layer) {
    return (int)(fold_of(h, layer, h->nc[layer]) % h->NB);
}
int *fold_ranks(iskv_handle *h, int layer, long long j) {
    return &h->fk[((size_t)layer * h->NB + (size_t)(j % h->NB)) * 4];
}

// Launches fold j (rows j*b .. j*b+b-1) of layers l0 .. l0+nl-1 on stream s: projection,
// residual basis, core SVD, basis update into buffer (j+1) % NB, Sigma into (j+1) % NB, H_top
// into j % NB and the new rows' coordinates. The history is rotated when the fold is applied.
int launch_fold_j(iskv_handle *h, int l0, int nl, long long j, cudaStream_t s) {
    const iskv_config &c = h->cfg;
    // the new rows' coordinates go to the block's rows, which must lie within n_max
    const long long nc = block_start(h, l0, j);
    if (nc + c.block > h->n_max) return ISKV_ERR_CAPACITY;
    const int bi = (int)(j % h->NB), bo = (int)((j + 1) % h->NB);
    // paths that run the regular update (a contiguous range: frozen paths are a prefix or suffix)
    const bool fz[2] = {frozen(h, 0, j), frozen(h, 1, j)};
    const int plo = fz[0] ? 1 : 0, phi = fz[1] ? 1 : 2;
    FoldArgs fa;
    memset(&fa, 0, sizeof(fa));
    fa.path_lo = plo;
    fa.path_hi = phi > plo ? phi : plo;
    for (int x = 0; x < 2; ++x) {
        const int r = rank_of(h, x);
        const int k = h->kf[x][l0];
        const int dj = h->joint ? c.n_kv_heads * D : D;     // columns of the factorised rows
        const int p = fz[x] ? 0 : (c.block < dj - k ? c.block : dj - k);
        const int kp = r < k + p ? r : k + p;
        FoldPath &fp = fa.path[x];
        fp.ring = h->ring[x];
        fp.basis_in = basis_buf(h, x, bi);
        fp.basis_out = basis_buf(h, x, bo);
        fp.sigma_in = sigma_buf(h, x, bi);
        fp.sigma_out = sigma_buf(h, x, bo);
        fp.coords = h->coords[x];
        fp.htop = htop_buf(h, x, bi);
        fp.r = r;
        fp.k = k;
        fp.p = p;
        fp.kp = kp;
    }
    fa.unit0 = l0 * h->UL;
    fa.n_c = nc;
    fa.n_max = h->n_max;
    fa.slot0 = (int)(nc % h->R);
    fa.R = h->R;
    fa.b = c.block;
    fa.kv_dtype = c.kv_dtype;
    fa.status = h->status;
    fa.stats = h->stats;
    fa.cbf = h->cbf;
    // coordinates of the block's real rows in the new basis (large blocks) or, for frozen paths,
    // in the frozen basis
    NewRowsArgs nr;
    memset(&nr, 0, sizeof(nr));
    for (int x = 0; x < 2; ++x) {
        nr.path[x].ring = h->ring[x];
        nr.path[x].basis = fz[x] ? fa.path[x].basis_in : fa.path[x].basis_out;
        nr.path[x].coords = h->coords[x];
        nr.path[x].r = fa.path[x].r;
        nr.path[x].kp = fa.path[x].kp;
    }
    nr.unit0 = fa.unit0;
    nr.slot0 = fa.slot0;
    nr.R = h->R;
    nr.b = c.block;
    nr.kv_dtype = c.kv_dtype;
    nr.n_c = nc;
    nr.n_max = h->n_max;
    nr.cbf = h->cbf;
    if (h->joint) {
        // one factorisation per (layer, sequence): the tall-skinny QR over the kv-heads, the fold
        // in the coordinates of [B P], then the kv-heads' slices of B+ = [B P] B~+
        JointArgs ja;
        memset(&ja, 0, sizeof(ja));
        for (int x = 0; x < 2; ++x) {
            JointPath &jp = ja.path[x];
            jp.ring = h->ring[x];
            jp.basis_in = fa.path[x].basis_in;
            jp.basis_out = fa.path[x].basis_out;
            jp.blk = h->jblk[x];
            jp.pbasis = h->jpb[x];
            jp.pbasis_out = h->jpbo[x];
            jp.refl = h->jrefl[x];
            jp.tau = h->jtau[x];
            jp.r = fa.path[x].r;
            jp.k = fa.path[x].k;
            jp.kp = fa.path[x].kp;
            fa.path[x].ring = h->jblk[x];
            fa.path[x].basis_in = h->jpb[x];
            fa.path[x].basis_out = h->jpbo[x];
        }
        ja.junit0 = l0 * h->JL;
        ja.H = c.n_kv_heads;
        ja.ldr = h->ldr;
        ja.slot0 = fa.slot0;
        ja.R = h->R;
        ja.b = c.block;
        ja.kv_dtype = c.kv_dtype;
        ja.path_lo = 0;
        ja.path_hi = 2;
        fa.unit0 = ja.junit0;
        fa.slot0 = 0;
        fa.R = c.block;
        fa.kv_dtype = ISKV_F32;
        if (launch_joint_prep(ja, nl * h->JL, s) != cudaSuccess ||
            launch_fold(fa, nl * h->JL, s) != cudaSuccess ||
            launch_joint_basis(ja, nl * h->JL, s) != cudaSuccess)
            return ISKV_ERR_CUDA;
        h->launches += 3;
    } else if (c.block > BMAX) {
        // large block: fold the 128-row triangular factor of the block (same Sigma+, H and basis),
        // then the coordinates of the block's real rows
        RFactorArgs rf;
        memset(&rf, 0, sizeof(rf));
        for (int x = 0; x < 2; ++x) {
            rf.path[x].ring = h->ring[x];
            rf.path[x].rout = h->rbig[x];
            fa.path[x].ring = h->rbig[x];
        }
        rf.unit0 = fa.unit0;
        rf.slot0 = fa.slot0;
        rf.R = h->R;
        rf.b = c.block;
        rf.kv_dtype = c.kv_dtype;
        rf.path_lo = fa.path_lo;
        rf.path_hi = fa.path_hi;
        if (launch_rfactor(rf, nl * h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        fa.slot0 = 0;
        fa.R = DEC_TILE;
        fa.b = DEC_TILE;
        fa.kv_dtype = ISKV_F32;
        fa.skip_new_rows = 1;
        if (launch_fold(fa, nl * h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        nr.path_lo = 0;
        nr.path_hi = 2;
        if (launch_newrows(nr, nl * h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        h->launches += (fa.path_hi > fa.path_lo ? 2 : 0) + 1;
    } else {
        if (launch_fold(fa, nl * h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        h->launches += fa.path_hi > fa.path_lo ? 1 : 0;
        if (fz[0] || fz[1]) {
            nr.path_lo = fz[0] ? 0 : 1;
            nr.path_hi = fz[1] ? 2 : 1;
            if (launch_newrows(nr, nl * h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
            h->launches += 1;
        }
    }
    // frozen paths carry their basis and Sigma over to the next fold's buffer
    for (int x = 0; x < 2; ++x) {
        if (!fz[x]) continue;
        const size_t r = (size_t)rank_of(h, x), u0 = (size_t)l0 * h->UL, nu = (size_t)nl * h->UL;
        if (cudaMemcpyAsync(basis_buf(h, x, bo) + u0 * D * r, basis_buf(h, x, bi) + u0 * D * r,
                            nu * D * r * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(sigma_buf(h, x, bo) + u0 * r, sigma_buf(h, x, bi) + u0 * r,
                            nu * r * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return ISKV_ERR_CUDA;
    }
    for (int l = l0; l < l0 + nl; ++l) {
        int *f = fold_ranks(h, l, j);
        f[0] = fa.path[0].k;
        f[1] = fa.path[0].kp;
        f[2] = fa.path[1].k;
        f[3] = fa.path[1].kp;
        h->kf[0][l] = fa.path[0].kp;
        h->kf[1][l] = fa.path[1].kp;
        h->nf[l] = j + 1;
    }
    return ISKV_OK;
}

// Applies the oldest pending fold of layers l0 .. l0+nl-1 on stream s: launches it here if no
// earlier call did, else makes s wait for it; then rotates the history C[0:n_c] <- C H_top and
// advances n_c, the ranks and the current buffer.
int apply_fold(iskv_handle *h, int l0, int nl, cudaStream_t s) {
    const iskv_config &c = h->cfg;
    const long long j = fold_of(h, l0, h->nc[l0]);
    const int bi = (int)(j % h->NB);
    if (h->nf[l0] <= j) {
        const int rc = launch_fold_j(h, l0, nl, j, s);
        if (rc != ISKV_OK) return rc;
        for (int l = l0; l < l0 + nl; ++l) h->on_side[(size_t)l * h->NB + bi] = 0;
    } else if (h->on_side[(size_t)l0 * h->NB + bi]) {
        if (cudaStreamWaitEvent(s, h->done[(size_t)l0 * h->NB + bi], 0) != cudaSuccess)
            return ISKV_ERR_CUDA;
        for (int l = l0; l < l0 + nl; ++l) h->on_side[(size_t)l * h->NB + bi] = 0;
    }
    const int *f = fold_ranks(h, l0, j);
    const long long nc = h->nc[l0];
    // frozen paths (fixed-basis mode) keep their old coordinates: nothing to rotate
    const bool fz[2] = {frozen(h, 0, j), frozen(h, 1, j)};
    if (nc > 0 && !(fz[0] && fz[1])) {
        RotArgs ra;
        memset(&ra, 0, sizeof(ra));
        ra.path_lo = fz[0] ? 1 : 0;
        ra.path_hi = fz[1] ? 1 : 2;
        for (int x = 0; x < 2; ++x) {
            RotPath &rp = ra.path[x];
            rp.coords = h->coords[x];
            rp.htop = htop_buf(h, x, bi);
            rp.r = rank_of(h, x);
            rp.k = f[2 * x];
            rp.kp = f[2 * x + 1];
        }
        ra.unit0 = l0 * h->CL;
        ra.n_old = nc;
        ra.n_max = h->n_max;
        ra.stale = c.rotate_history ? 0 : 1;
        ra.cbf = h->cbf;
        if (launch_rotate(ra, nl * h->CL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        h->launches += 1;
    }
    for (int l = l0; l < l0 + nl; ++l) {
        h->nc[l] += c.block;
        h->kcur[0][l] = f[1];
        h->kcur[1][l] = f[3];
    }
    return ISKV_OK;
}

// Look-ahead: starts every fold whose block is complete on an internal stream (forked from s),
// as far as the buffer ring allows and only for blocks that the window can still release within
// max_tokens (the others are never applied, and their coordinates would not fit in n_max rows);
// apply_fold() later joins it back.
int launch_ahead(iskv_handle *h, int l0, int nl, cudaStream_t s) {
    const iskv_config &c = h->cfg;
    cudaStream_t side = h->side[l0 % iskv_handle::NS];
    bool forked = false;
    while (block_start(h, l0, h->nf[l0]) + c.block <= h->t[l0] &&
           block_start(h, l0, h->nf[l0]) + c.block <= h->n_max &&
           h->nf[l0] <= fold_of(h, l0, h->nc[l0]) + h->NB - 2) {
        const long long j = h->nf[l0];
        const int bi = (int)(j % h->NB);
        if (!forked) {
            if (cudaEventRecord(h->fork, s) != cudaSuccess ||
                cudaStreamWaitEvent(side, h->fork, 0) != cudaSuccess)
                return ISKV_ERR_CUDA;
            forked = true;
        }
        const int rc = launch_fold_j(h, l0, nl, j, side);
        if (rc != ISKV_OK) return rc;
        for (int l = l0; l < l0 + nl; ++l) {
            if (cudaEventRecord(h->done[(size_t)l * h->NB + bi], side) != cudaSuccess)
                return ISKV_ERR_CUDA;
            h->on_side[(size_t)l * h->NB + bi] = 1;
        }
    }
    return ISKV_OK;
}

// Makes s wait for every fold still running on an internal stream.
int join_all(iskv_handle *h, cudaStream_t s) {
    for (int l = 0; l < h->cfg.n_layers; ++l)
        for (int i = 0; i < h->NB; ++i) {
            unsigned char &f = h->on_side[(size_t)l * h->NB + i];
            if (!f) continue;
            if (cudaStreamWaitEvent(s, h->done[(size_t)l * h->NB + i], 0) != cudaSuccess)
                return ISKV_ERR_CUDA;
            f = 0;
        }
    return ISKV_OK;
}

}  // namespace

extern "C" {

const char *iskv_strerror(int code) {
    switch (code) {
        case ISKV_OK: return "ok";
        case ISKV_ERR_INVALID_ARG: return "invalid argument";
        case ISKV_ERR_CAPACITY: return "capacity exceeded (t + m > max_tokens)";
        case ISKV_ERR_CUDA: return "CUDA runtime error";
        case ISKV_ERR_NOT_CONVERGED: return "core SVD did not converge within the sweep cap";
        case ISKV_ERR_NONFINITE: return "non-finite singular value";
        case ISKV_ERR_UNSUPPORTED: return "unsupported configuration";
        case ISKV_ERR_TIMEOUT: return "a device-side wait exceeded its bound";
        default: return "unknown error";
    }
}

int iskv_schedule(int block, int window, long long t, long long m, long long *n_c_out,
                  long long *folds_out) {
    if (block < 1 || window < 0 || t < 0 || m < 0) return ISKV_ERR_INVALID_ARG;
    const long long a = ncomp(t, block, window), b = ncomp(t + m, block, window);
    if (n_c_out) *n_c_out = b;
    if (folds_out) *folds_out = (b - a) / block;
    return ISKV_OK;
}

int iskv_create(const iskv_config *cfg, iskv_handle **out) {
    if (!cfg || !out) return ISKV_ERR_INVALID_ARG;
    *out = nullptr;
    const iskv_config &c = *cfg;
    if (c.batch < 1 || c.n_layers < 1 || c.n_kv_heads < 1 || c.n_q_heads < c.n_kv_heads ||
        c.n_q_heads % c.n_kv_heads != 0 || c.n_q_heads / c.n_kv_heads > GMAX || c.head_dim != D ||
        c.rank_k < 1 || c.rank_k > D || c.rank_v < 1 || c.rank_v > D || c.block < 1 ||
        c.window < 0 || c.max_tokens < 1 || (c.kv_dtype != ISKV_BF16 && c.kv_dtype != ISKV_F32) ||
        (c.rope && !(c.rope_theta > 0.0)) || (c.fixed_basis && !c.rotate_history) ||
        c.prot_cap < 0)
        return ISKV_ERR_INVALID_ARG;
    if (c.block > BMAX_LARGE) return ISKV_ERR_UNSUPPORTED;
    if (c.joint_heads && (c.rank_k + c.block > D || c.rank_v + c.block > D || c.fixed_basis ||
                          c.prot_cap > 0))
        return ISKV_ERR_UNSUPPORTED;
    iskv_handle *h = new (std::nothrow) iskv_handle();
    if (!h) return ISKV_ERR_CUDA;
    try {
        h->cfg = c;
        if (cudaGetDevice(&h->device) != cudaSuccess) {
            delete h;
            return ISKV_ERR_CUDA;
        }
        cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device);
        h->UL = c.batch * c.n_kv_heads;
        h->U = c.n_layers * h->UL;
        h->joint = c.joint_heads != 0;
        h->JL = c.batch;
        h->CL = h->joint ? c.batch : h->UL;
        h->CU = c.n_layers * h->CL;
        h->ldr = (c.rank_k > c.rank_v ? c.rank_k : c.rank_v) + c.block;
        h->R = c.window + c.block;
        h->G = c.n_q_heads / c.n_kv_heads;
        // compressed positions: up to max_tokens - window (a prefill's end need not be a
        // multiple of the block)
        h->n_max = c.max_tokens > c.window ? c.max_tokens - c.window : 0;
        h->pcap = c.prot_cap;
        h->esz = c.kv_dtype == ISKV_BF16 ? 2 : 4;
        h->cbf = c.coord_bf16 ? 1 : 0;
        h->csz = h->cbf ? 2 : 4;
        const long long ctiles = (h->n_max + DEC_TILE - 1) / DEC_TILE;
        h->max_splits = (int)(ctiles + (h->R + DEC_TILE - 1) / DEC_TILE + 1);
        // folds in flight ahead of their trigger: at most window / block + 1 (look-ahead only)
        h->NB = c.lookahead_folds ? c.window / c.block + 3 : 2;
        h->t.assign(c.n_layers, 0);
        h->nc.assign(c.n_layers, 0);
        h->nf.assign(c.n_layers, 0);
        h->pbase.assign(c.n_layers, 0);
        h->pfold.assign(c.n_layers, 0);
        h->ptiles.assign(c.n_layers, 0);
        h->pact.assign(c.n_layers, 0);
        for (int x = 0; x < 2; ++x) {
            h->kcur[x].assign(c.n_layers, 0);
            h->kf[x].assign(c.n_layers, 0);
        }
        h->fk.assign((size_t)c.n_layers * h->NB * 4, 0);
        h->on_side.assign((size_t)c.n_layers * h->NB, 0);
        h->done.assign((size_t)c.n_layers * h->NB, nullptr);
    } catch (...) {
        delete h;
        return ISKV_ERR_CUDA;
    }
    bool ok = true;
    auto alloc = [&](void **p, size_t bytes) {
        if (!ok) return;
        if (bytes == 0) bytes = 16;
        if (cudaMalloc(p, bytes) != cudaSuccess) {
            ok = false;
            *p = nullptr;
        }
    };
    const size_t U = (size_t)h->U;
    for (int x = 0; x < 2; ++x) {
        const size_t r = (size_t)rank_of(h, x);
        const size_t nb = (size_t)h->NB;
        alloc((void **)&h->coords[x], (size_t)h->CU * (size_t)h->n_max * r * h->csz);
        if (h->joint) {
            const size_t J = (size_t)h->CU, Hk = (size_t)c.n_kv_heads;
            alloc((void **)&h->jblk[x], J * c.block * D * sizeof(float));
            alloc((void **)&h->jpb[x], J * D * r * sizeof(float));
            alloc((void **)&h->jpbo[x], J * D * r * sizeof(float));
            alloc((void **)&h->jrefl[x], J * Hk * D * h->ldr * sizeof(float));
            alloc((void **)&h->jtau[x], J * Hk * h->ldr * sizeof(float));
        }
        alloc((void **)&h->basis[x], nb * U * D * r * sizeof(float));
        alloc((void **)&h->sigma[x], nb * U * r * sizeof(float));
        alloc(&h->ring[x], U * (size_t)h->R * D * h->esz);
        alloc((void **)&h->htop[x], nb * U * r * r * sizeof(float));
        if (c.block > BMAX || c.prot_cap > 0)
            alloc((void **)&h->rbig[x], U * DEC_TILE * D * sizeof(float));
        if (c.prot_cap > 0) {
            alloc((void **)&h->ppos[x], U * (size_t)c.prot_cap * sizeof(int));
            alloc(&h->pstore[x], U * (size_t)c.prot_cap * D * h->esz);
            alloc((void **)&h->pcount[x], U * sizeof(int));
        }
    }
    if (c.rope) alloc((void **)&h->rope_cs, (size_t)c.max_tokens * DH * sizeof(float2));
    if (c.rope) alloc((void **)&h->rope_t, (size_t)c.max_tokens * DH * sizeof(float2));
    {
        // split partials: the larger of the split-kernel layout and the persistent decode's
        const size_t a1 = (size_t)h->UL * h->max_splits * h->G * (2 + D);
        const size_t a2 = ws_partial_floats(h->UL, h->sms, h->G, c.rank_v);
        alloc((void **)&h->ws, (a1 > a2 ? a1 : a2) * sizeof(float));
    }
    alloc((void **)&h->status, sizeof(int));
    if (c.prot_cap > 0) {
        alloc((void **)&h->pflags, U * (size_t)(h->n_max > 0 ? h->n_max : 1));
        alloc((void **)&h->pscores, (size_t)h->UL * (size_t)(h->n_max > 0 ? h->n_max : 1) * sizeof(float));
    }
    alloc((void **)&h->stats, 4 * sizeof(unsigned long long));
    if (ok) {
        for (int x = 0; x < 2; ++x) {
            const size_t r = (size_t)rank_of(h, x), nb = (size_t)h->NB;
            ok = ok && cudaMemset(h->basis[x], 0, nb * U * D * r * sizeof(float)) == cudaSuccess;
            ok = ok && cudaMemset(h->sigma[x], 0, nb * U * r * sizeof(float)) == cudaSuccess;
        }
        ok = ok && cudaMemset(h->status, 0, sizeof(int)) == cudaSuccess;
        if (ok && c.prot_cap > 0) {
            ok = cudaMemset(h->pflags, 0, U * (size_t)(h->n_max > 0 ? h->n_max : 1)) == cudaSuccess &&
                 cudaMemset(h->pcount[0], 0, U * sizeof(int)) == cudaSuccess &&
                 cudaMemset(h->pcount[1], 0, U * sizeof(int)) == cudaSuccess;
        }
        ok = ok && cudaMemset(h->stats, 0, 4 * sizeof(unsigned long long)) == cudaSuccess;
        for (int i = 0; ok && i < iskv_handle::NS; ++i)
            ok = cudaStreamCreateWithFlags(&h->side[i], cudaStreamNonBlocking) == cudaSuccess;
        ok = ok && cudaEventCreateWithFlags(&h->fork, cudaEventDisableTiming) == cudaSuccess;
        for (size_t i = 0; ok && i < h->done.size(); ++i)
            ok = cudaEventCreateWithFlags(&h->done[i], cudaEventDisableTiming) == cudaSuccess;
        if (ok && c.rope)
            ok = launch_rope_table(h->rope_cs, c.max_tokens, c.rope_theta, 0) == cudaSuccess &&
                 launch_rope_table_t(h->rope_t, c.max_tokens, c.rope_theta, 0) == cudaSuccess;
        ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    }
    if (!ok) {
        free_all(h);
        delete h;
        cudaGetLastError();
        return ISKV_ERR_CUDA;
    }
    // tensor-core decode: key coordinates in 32-column TMA boxes (r_K <= 64, rows 16-byte
    // aligned), value rows copied in bulk (r_V multiple of 4), compute capability 10.x
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, h->device);
    memset(&h->tmC, 0, sizeof(h->tmC));
    memset(&h->tmB, 0, sizeof(h->tmB));
    if (h->cbf) {
        // bf16 coordinates are read by the persistent decode only: one 64-column box of key
        // coordinates, 16-byte rows of value coordinates
        bool m_ok = major == 10 && c.rank_k % 8 == 0 && c.rank_k <= 64 && c.rank_v % 8 == 0 &&
                    (h->G == 1 || h->G == 2 || h->G == 4) &&
                    ws_smem_bytes(1, c.rank_v, (int)h->esz, h->G) <= 227 * 1024;
        if (m_ok && h->n_max > 0)
            m_ok = make_map(&h->tmC, h->coords[0], c.rank_k, (long long)h->CU * h->n_max, true);
        if (!m_ok) {
            free_all(h);
            delete h;
            return ISKV_ERR_UNSUPPORTED;
        }
        h->tc = h->ws_ok = true;
    } else if (major == 10 && c.rank_k % 4 == 0 && c.rank_k <= 64 && c.rank_v % 4 == 0 &&
               tc_smem_bytes((c.rank_k + 31) / 32, c.rank_v, (int)h->esz, h->G) <= 227 * 1024) {
        bool m_ok = true;
        if (h->n_max > 0) {
            m_ok = make_map(&h->tmC, h->coords[0], c.rank_k, (long long)h->CU * h->n_max) &&
                   make_map(&h->tmB, h->basis[0], c.rank_k, (long long)h->NB * h->U * D);
        }
        h->tc = m_ok;
        // persistent warp-specialised decode: fp32 key coordinates in one 32-column box, GQA
        // groups of 1, 2 or 4, value rows in 16-byte units
        h->ws_ok = m_ok && c.rank_k <= 32 && (h->G == 1 || h->G == 2 || h->G == 4) &&
                   ws_smem_bytes(0, c.rank_v, (int)h->esz, h->G) <= 227 * 1024;
    }
    *out = h;
    return ISKV_OK;
}

int iskv_destroy(iskv_handle *h) {
    if (!h) return ISKV_OK;
    DeviceGuard g(h->device);
    cudaDeviceSynchronize();
    free_all(h);
    delete h;
    return ISKV_OK;
}

int iskv_append_block(iskv_handle *h, int layer, const void *k_rows, const void *v_rows, int m,
                      iskv_stream_t stream) {
    if (!h || !k_rows || !v_rows || m < 1) return ISKV_ERR_INVALID_ARG;
    const iskv_config &c = h->cfg;
    if (layer != -1 && !valid_layer(h, layer)) return ISKV_ERR_INVALID_ARG;
    const int l0 = layer < 0 ? 0 : layer;
    const int nl = layer < 0 ? c.n_layers : 1;
    for (int l = l0; l < l0 + nl; ++l)
        if (h->t[l] != h->t[l0] || h->nc[l] != h->nc[l0] || h->nf[l] != h->nf[l0])
            return ISKV_ERR_INVALID_ARG;
    if (h->t[l0] + m > c.max_tokens) return ISKV_ERR_CAPACITY;
    DeviceGuard g(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    long long t = h->t[l0];
    int done = 0;
    while (done < m) {
        const long long e = t - h->nc[l0];
        const long long room = (long long)h->R - e;   // rows until the window holds w + b
        const int chunk = (int)((long long)(m - done) < room ? (m - done) : room);
        AppendArgs aa;
        aa.src[0] = k_rows;
        aa.src[1] = v_rows;
        aa.ring[0] = h->ring[0];
        aa.ring[1] = h->ring[1];
        aa.unit0 = l0 * h->UL;
        aa.m_total = m;
        aa.row0 = done;
        aa.rows = chunk;
        aa.pos0 = t;
        aa.R = h->R;
        aa.kv_dtype = c.kv_dtype;
        if (launch_append(aa, nl * h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        h->launches += 1;
        t += chunk;
        done += chunk;
        for (int l = l0; l < l0 + nl; ++l) h->t[l] = t;
        if (t - h->nc[l0] >= (long long)h->R) {
            const int rc = apply_fold(h, l0, nl, s);
            if (rc != ISKV_OK) return rc;
        }
        if (c.lookahead_folds) {
            const int rc = launch_ahead(h, l0, nl, s);
            if (rc != ISKV_OK) return rc;
        }
    }
    return ISKV_OK;
}

}  // extern "C"

namespace {

// Decode attention of one layer over positions 0 .. t-1. With new_k/new_v (tensor-core path),
// the row of position t-1 is taken from the caller's arrays and stored in the ring by the kernel.
int decode_layer(iskv_handle *h, int layer, const float *q, float *out, cudaStream_t s,
                 const void *new_k, const void *new_v) {
    const iskv_config &c = h->cfg;
    DecodeArgs da;
    memset(&da, 0, sizeof(da));
    const int cur = current_buffer(h, layer);
    for (int x = 0; x < 2; ++x) {
        const size_t r = (size_t)rank_of(h, x);
        const size_t u0 = (size_t)layer * h->UL, c0 = (size_t)layer * h->CL;
        da.coords[x] = static_cast<const char *>(h->coords[x]) + c0 * (size_t)h->n_max * r * h->csz;
        da.basis[x] = basis_buf(h, x, cur) + u0 * D * r;
        da.ring[x] = static_cast<const char *>(h->ring[x]) + u0 * (size_t)h->R * D * h->esz;
        da.r[x] = (int)r;
        da.k[x] = h->kcur[x][layer];
    }
    da.rope_cs = c.rope ? h->rope_cs : nullptr;
    da.q = q;
    da.out = out;
    da.ws = h->ws;
    da.n_c = h->nc[layer];
    da.t = h->t[layer];
    da.n_max = h->n_max;
    da.R = h->R;
    da.H = c.n_kv_heads;
    da.G = h->G;
    da.new_row[0] = new_k;
    da.new_row[1] = new_v;
    da.new_pos = new_k ? da.t - 1 : -1;
    da.cbf = h->cbf;
    da.cdiv = h->joint ? c.n_kv_heads : 1;
    // compressed splits: at most one wave of CTAs over all units of the layer (two per SM when
    // two fit in shared memory), the compressed tiles of a unit spread evenly over its splits
    const long long ctiles = (da.n_c + DEC_TILE - 1) / DEC_TILE;
    const int per_sm = (!h->tc || tc_smem_bytes((c.rank_k + 31) / 32, c.rank_v, (int)h->esz, h->G) +
                                          1024 <= 114u * 1024u) ? 2 : 1;
    long long per_unit = (long long)per_sm * h->sms / h->UL;
    if (per_unit < 1) per_unit = 1;
    const long long nsc = ctiles < per_unit ? ctiles : per_unit;
    const long long tps = nsc > 0 ? (ctiles + nsc - 1) / nsc : 1;
    da.split_rows = (int)(tps * DEC_TILE);
    da.n_split_c = (int)((ctiles + tps - 1) / tps);
    const long long e = da.t - da.n_c;
    da.n_split = da.n_split_c + (int)((e + DEC_TILE - 1) / DEC_TILE);
    da.max_splits = h->max_splits;
    da.kv_dtype = c.kv_dtype;
    da.scale = 1.0f / sqrtf((float)D);
    // the persistent decode pays off once every SM streams several tiles; smaller calls (fp32
    // coordinates, no protection) use the split-kernel decode
    const long long tiles_ws = (long long)h->UL * (ctiles + (e + DEC_TILE - 1) / DEC_TILE);
    const bool use_ws = h->ws_ok && (h->cbf || h->pact[layer] || !h->tc ||
                                     tiles_ws >= 6LL * h->sms);
    if (use_ws) {
        if (reinterpret_cast<uintptr_t>(q) % 16 != 0) return ISKV_ERR_INVALID_ARG;
        WsExtra x;
        memset(&x, 0, sizeof(x));
        x.rope_rows = c.max_tokens;
        x.row0 = (long long)layer * h->CL * h->n_max;
        x.brow0 = (cur * h->U + layer * h->UL) * D;
        x.Tc = (int)ctiles;
        x.Tw = (int)((e + DEC_TILE - 1) / DEC_TILE);
        // an exact-row tile (keys read and rotated on CUDA cores, values summed over 128 channels)
        // costs several compressed tiles: it takes four slots of the CTAs' equal shares (measured
        // best of 2 .. 6 on the 64-unit 32K-token and the 8-unit 16K-token layer calls)
        x.W = 4;
        x.Tu = x.Tc + x.W * x.Tw;
        x.UL = h->UL;
        x.N = (long long)h->UL * x.Tu;
        x.P = (int)(x.N < h->sms ? x.N : h->sms);
        x.maxseg = h->UL / x.P + 2;
        x.factor_bf16 = h->cbf;
        x.status = h->status;
        if (h->pact[layer]) {
            const size_t u0 = (size_t)layer * h->UL;
            x.pflags = h->pflags + u0 * (size_t)h->n_max;
            x.fstride = h->n_max;
            for (int p = 0; p < 2; ++p) {
                x.ppos[p] = h->ppos[p] + u0 * h->pcap;
                x.pstore[p] = static_cast<const char *>(h->pstore[p]) + u0 * h->pcap * D * h->esz;
                x.pcount[p] = h->pcount[p] + u0;
            }
            x.pcap = h->pcap;
            x.Tp = h->ptiles[layer];
            x.Tu = x.Tc + x.W * (x.Tp + x.Tw);
            x.N = (long long)h->UL * x.Tu;
            x.P = (int)(x.N < h->sms ? x.N : h->sms);
            x.maxseg = h->UL / x.P + 2;
        }
        if (x.N < 1) return ISKV_ERR_INVALID_ARG;
        const cudaError_t e = launch_decode_ws(&h->tmC, &h->tmB, da, x, s);
        if (e == cudaSuccess) {
            h->launches += 2;
            return ISKV_OK;
        }
        // a build whose register allocation cannot hold the kernel's register split is never
        // launched: use the split-kernel decode from now on (fp32 coordinates, no protection)
        if (e != cudaErrorInvalidConfiguration || h->cbf || h->pact[layer]) return ISKV_ERR_CUDA;
        h->ws_ok = false;
    }
    if (da.n_split > h->max_splits) return ISKV_ERR_INVALID_ARG;
    if (h->tc) {
        if (reinterpret_cast<uintptr_t>(q) % 16 != 0) return ISKV_ERR_INVALID_ARG;
        TcExtra x;
        x.kblocks = (c.rank_k + 31) / 32;
        x.row0 = (long long)layer * h->CL * h->n_max;
        x.brow0 = (cur * h->U + layer * h->UL) * D;
        x.rope_t = c.rope ? h->rope_t : nullptr;
        x.rope_rows = c.max_tokens;
        x.status = h->status;
        if (launch_decode_tc(&h->tmC, &h->tmB, da, x, h->UL, s) != cudaSuccess)
            return ISKV_ERR_CUDA;
        h->launches += 2;
        return ISKV_OK;
    }
    if (new_k) return ISKV_ERR_UNSUPPORTED;     // callers fall back to a separate append
    if (launch_decode(da, h->UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
    h->launches += 2;
    return ISKV_OK;
}

}  // namespace

extern "C" {

int iskv_prefill(iskv_handle *h, int layer, const void *k_rows, const void *v_rows, long long T0,
                 const iskv_protect *prot, iskv_stream_t stream) {
    if (!h || !k_rows || !v_rows || !valid_layer(h, layer) || T0 < 1) return ISKV_ERR_INVALID_ARG;
    const iskv_config &c = h->cfg;
    if (h->t[layer] != 0 || h->nf[layer] != 0) return ISKV_ERR_INVALID_ARG;
    if (prot && (prot->chunk < 1 || prot->m < 0 || prot->suffix < 0 || prot->rho < 0))
        return ISKV_ERR_INVALID_ARG;
    if (T0 > c.max_tokens) return ISKV_ERR_CAPACITY;
    if (h->pcap <= 0) return ISKV_ERR_UNSUPPORTED;
    const long long end = T0 - c.window;
    if (end <= 0) return iskv_append_block(h, layer, k_rows, v_rows, (int)T0, stream);
    if (end > 0x7fffffffLL) return ISKV_ERR_UNSUPPORTED;
    if (prot && !h->ws_ok) return ISKV_ERR_UNSUPPORTED;
    const int n_chunks = prot ? (int)((end + prot->chunk - 1) / prot->chunk) : 0;
    if (prot && (prot_select_smem(n_chunks, prot->m < n_chunks ? prot->m : n_chunks) > 227 * 1024 ||
                 prot_score_smem(prot->chunk) > 227 * 1024))
        return ISKV_ERR_UNSUPPORTED;               // too many chunks (or too long a chunk) for one CTA
    DeviceGuard g(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int UL = h->UL, u0 = layer * UL;
    // 1-2. protected positions and stores (step 1 for keys, step 2 for values)
    if (prot) {
        ProtArgs pa;
        memset(&pa, 0, sizeof(pa));
        pa.keys = k_rows;
        pa.src[0] = k_rows;
        pa.src[1] = v_rows;
        pa.src_rows = T0;
        pa.end = end;
        pa.T0 = T0;
        pa.chunk = prot->chunk;
        pa.n_chunks = (int)((end + prot->chunk - 1) / prot->chunk);
        pa.m = prot->m < pa.n_chunks ? prot->m : pa.n_chunks;      // "up to m" chunks
        pa.suffix = prot->suffix;
        pa.rho = prot->rho;
        pa.n_chunks_cap = (int)h->n_max;
        pa.scores = h->pscores;
        pa.flags = h->pflags;
        pa.flag_stride = h->n_max;
        pa.unit0 = u0;
        pa.cap = h->pcap;
        for (int x = 0; x < 2; ++x) {
            pa.ppos[x] = h->ppos[x];
            pa.store[x] = h->pstore[x];
            pa.pcount[x] = h->pcount[x];
        }
        pa.rope_cs = c.rope ? h->rope_cs : nullptr;
        pa.kv_dtype = c.kv_dtype;
        pa.status = h->status;
        if (launch_protect(pa, UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
        h->launches += 2;
    }
    // 3. truncated SVD of the remaining rows: their triangular factor, then its fold from rank 0
    RFactorArgs rf;
    memset(&rf, 0, sizeof(rf));
    for (int x = 0; x < 2; ++x) {
        rf.path[x].rout = h->rbig[x];
        rf.path[x].src = x ? v_rows : k_rows;
        rf.path[x].fbit = prot ? (1 << x) : 0;
    }
    rf.unit0 = u0;
    rf.R = 1;
    rf.b = (int)end;
    rf.kv_dtype = c.kv_dtype;
    rf.path_lo = 0;
    rf.path_hi = 2;
    rf.src_rows = T0;
    rf.flags = h->pflags;
    rf.flag_stride = h->n_max;
    if (!prot) rf.flags = nullptr;
    if (launch_rfactor(rf, UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
    FoldArgs fa;
    memset(&fa, 0, sizeof(fa));
    int kp[2];
    for (int x = 0; x < 2; ++x) {
        const int r = rank_of(h, x);
        kp[x] = r < DEC_TILE ? r : DEC_TILE;
        FoldPath &fp = fa.path[x];
        fp.ring = h->rbig[x];
        fp.basis_in = basis_buf(h, x, 0);
        fp.basis_out = basis_buf(h, x, 1);
        fp.sigma_in = sigma_buf(h, x, 0);
        fp.sigma_out = sigma_buf(h, x, 1);
        fp.coords = h->coords[x];
        fp.htop = htop_buf(h, x, 0);
        fp.r = r;
        fp.k = 0;
        fp.p = DEC_TILE;
        fp.kp = kp[x];
    }
    fa.unit0 = u0;
    fa.n_c = 0;
    fa.n_max = h->n_max;
    fa.slot0 = 0;
    fa.R = DEC_TILE;
    fa.b = DEC_TILE;
    fa.kv_dtype = ISKV_F32;
    fa.status = h->status;
    fa.stats = h->stats;
    fa.skip_new_rows = 1;
    fa.path_lo = 0;
    fa.path_hi = 2;
    fa.cbf = h->cbf;
    if (launch_fold(fa, UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
    // coordinates of every row before the window (zero for protected rows)
    NewRowsArgs nr;
    memset(&nr, 0, sizeof(nr));
    for (int x = 0; x < 2; ++x) {
        nr.path[x].basis = basis_buf(h, x, 1);
        nr.path[x].coords = h->coords[x];
        nr.path[x].r = rank_of(h, x);
        nr.path[x].kp = kp[x];
        nr.path[x].src = x ? v_rows : k_rows;
        nr.path[x].fbit = prot ? (1 << x) : 0;
    }
    nr.unit0 = u0;
    nr.R = 1;
    nr.b = (int)end;
    nr.kv_dtype = c.kv_dtype;
    nr.n_c = 0;
    nr.n_max = h->n_max;
    nr.path_lo = 0;
    nr.path_hi = 2;
    nr.cbf = h->cbf;
    nr.src_rows = T0;
    nr.flags = prot ? h->pflags : nullptr;
    nr.flag_stride = h->n_max;
    if (launch_newrows(nr, UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
    // the window: rows end .. T0 - 1
    AppendArgs aa;
    aa.src[0] = k_rows;
    aa.src[1] = v_rows;
    aa.ring[0] = h->ring[0];
    aa.ring[1] = h->ring[1];
    aa.unit0 = u0;
    aa.m_total = (int)T0;
    aa.row0 = (int)end;
    aa.rows = (int)(T0 - end);
    aa.pos0 = end;
    aa.R = h->R;
    aa.kv_dtype = c.kv_dtype;
    if (launch_append(aa, UL, s) != cudaSuccess) return ISKV_ERR_CUDA;
    h->launches += 4;
    // host state: the prefill is update 0 of the layer
    h->t[layer] = T0;
    h->nc[layer] = end;
    h->pbase[layer] = end;
    h->pfold[layer] = 1;
    h->nf[layer] = 1;
    for (int x = 0; x < 2; ++x) h->kcur[x][layer] = h->kf[x][layer] = kp[x];
    int *f = fold_ranks(h, layer, 0);
    f[0] = 0;
    f[1] = kp[0];
    f[2] = 0;
    f[3] = kp[1];
    if (prot) {
        // the largest protected key count sizes the decode's protected tiles
        std::vector<int> cnt(UL);
        if (cudaMemcpyAsync(cnt.data(), h->pcount[0] + u0, UL * sizeof(int), cudaMemcpyDeviceToHost,
                            s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return ISKV_ERR_CUDA;
        int mx = 0;
        for (int v : cnt) mx = v > mx ? v : mx;
        h->ptiles[layer] = (mx + DEC_TILE - 1) / DEC_TILE;
        h->pact[layer] = 1;
    }
    if (c.lookahead_folds) return launch_ahead(h, layer, 1, s);
    return ISKV_OK;
}

int iskv_decode_attn(iskv_handle *h, int layer, const float *q, float *out, iskv_stream_t stream) {
    if (!h || !q || !out || !valid_layer(h, layer)) return ISKV_ERR_INVALID_ARG;
    if (h->t[layer] < 1) return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    return decode_layer(h, layer, q, out, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr);
}

int iskv_append_decode(iskv_handle *h, int layer, const void *k_row, const void *v_row,
                       const float *q, float *out, iskv_stream_t stream) {
    if (!h || !k_row || !v_row || !q || !out || !valid_layer(h, layer)) return ISKV_ERR_INVALID_ARG;
    const iskv_config &c = h->cfg;
    // the fused form needs the tensor-core decode, and a window of at least one row (so that a
    // fold released by this token never needs the token's own row)
    if (!h->tc || c.window < 1) {
        int rc = iskv_append_block(h, layer, k_row, v_row, 1, stream);
        if (rc != ISKV_OK) return rc;
        return iskv_decode_attn(h, layer, q, out, stream);
    }
    if (h->t[layer] + 1 > c.max_tokens) return ISKV_ERR_CAPACITY;
    DeviceGuard g(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    h->t[layer] += 1;
    if (h->t[layer] - h->nc[layer] >= (long long)h->R) {
        const int rc = apply_fold(h, layer, 1, s);
        if (rc != ISKV_OK) return rc;
    }
    int rc = decode_layer(h, layer, q, out, s, k_row, v_row);
    if (rc != ISKV_OK) return rc;
    if (c.lookahead_folds) rc = launch_ahead(h, layer, 1, s);
    return rc;
}

int iskv_reconstruct(iskv_handle *h, int layer, int which, int apply_rope, float *out,
                     iskv_stream_t stream) {
    if (!h || !out || !valid_layer(h, layer) || (which != 0 && which != 1))
        return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    const size_t r = (size_t)rank_of(h, which);
    const size_t u0 = (size_t)layer * h->UL, c0 = (size_t)layer * h->CL;
    ReconArgs ra;
    memset(&ra, 0, sizeof(ra));
    ra.coords = static_cast<const char *>(h->coords[which]) + c0 * (size_t)h->n_max * r * h->csz;
    ra.cbf = h->cbf;
    ra.cdiv = h->joint ? h->cfg.n_kv_heads : 1;
    ra.basis = basis_buf(h, which, current_buffer(h, layer)) + u0 * D * r;
    ra.ring = static_cast<const char *>(h->ring[which]) + u0 * (size_t)h->R * D * h->esz;
    ra.rope_cs = h->rope_cs;
    ra.out = out;
    ra.r = (int)r;
    ra.k = h->kcur[which][layer];
    ra.n_c = h->nc[layer];
    ra.t = h->t[layer];
    ra.n_max = h->n_max;
    ra.R = h->R;
    ra.kv_dtype = h->cfg.kv_dtype;
    ra.apply_rope = (which == 0 && apply_rope && h->cfg.rope) ? 1 : 0;
    if (h->pact[layer]) {
        ra.pflags = h->pflags + u0 * (size_t)h->n_max;
        ra.fstride = h->n_max;
        ra.fbit = which ? 2 : 1;
        ra.ppos = h->ppos[which] + u0 * h->pcap;
        ra.pstore = static_cast<const char *>(h->pstore[which]) + u0 * h->pcap * D * h->esz;
        ra.pcount = h->pcount[which] + u0;
        ra.pcap = h->pcap;
    }
    if (launch_reconstruct(ra, h->UL, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ISKV_ERR_CUDA;
    h->launches += ra.t > 0 ? 1 : 0;
    return ISKV_OK;
}

int iskv_get_factors(iskv_handle *h, int layer, int seq, int kv_head, int which, float *coords,
                     float *basis, float *sigma, int *k_out, long long *n_c_out,
                     iskv_stream_t stream) {
    if (!h || !valid_layer(h, layer) || seq < 0 || seq >= h->cfg.batch || kv_head < 0 ||
        kv_head >= h->cfg.n_kv_heads || (which != 0 && which != 1))
        return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t r = (size_t)rank_of(h, which);
    const size_t u = ((size_t)layer * h->cfg.batch + seq) * h->cfg.n_kv_heads + kv_head;
    // coordinates, Sigma: the kv-head's unit, or the (layer, sequence)'s joint unit
    const size_t cu = h->joint ? (size_t)layer * h->cfg.batch + seq : u;
    const long long nc = h->nc[layer];
    if (coords && nc > 0) {
        const void *src = static_cast<const char *>(h->coords[which]) + cu * (size_t)h->n_max * r * h->csz;
        const cudaError_t e = h->cbf ? launch_coords_to_f32(coords, src, (size_t)nc * r, s)
                                     : cudaMemcpyAsync(coords, src, (size_t)nc * r * sizeof(float),
                                                       cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return ISKV_ERR_CUDA;
        h->launches += h->cbf ? 1 : 0;
    }
    const int cur = current_buffer(h, layer);
    if (basis && cudaMemcpyAsync(basis, basis_buf(h, which, cur) + u * D * r,
                                 D * r * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return ISKV_ERR_CUDA;
    if (sigma && cudaMemcpyAsync(sigma, sigma_buf(h, which, cur) + cu * r, r * sizeof(float),
                                 cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return ISKV_ERR_CUDA;
    if (k_out) *k_out = h->kcur[which][layer];
    if (n_c_out) *n_c_out = nc;
    return ISKV_OK;
}

int iskv_join(iskv_handle *h, iskv_stream_t stream) {
    if (!h) return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    return join_all(h, reinterpret_cast<cudaStream_t>(stream));
}

int iskv_reset(iskv_handle *h, iskv_stream_t stream) {
    if (!h) return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    const int rc = join_all(h, reinterpret_cast<cudaStream_t>(stream));
    if (rc != ISKV_OK) return rc;
    for (int l = 0; l < h->cfg.n_layers; ++l) {
        h->t[l] = 0;
        h->nc[l] = 0;
        h->nf[l] = 0;
        h->pbase[l] = 0;
        h->pfold[l] = 0;
        h->ptiles[l] = 0;
        h->pact[l] = 0;
        for (int x = 0; x < 2; ++x) h->kcur[x][l] = h->kf[x][l] = 0;
    }
    if (cudaMemsetAsync(h->status, 0, sizeof(int), reinterpret_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return ISKV_ERR_CUDA;
    if (h->pcap > 0) {
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (cudaMemsetAsync(h->pflags, 0, (size_t)h->U * (size_t)(h->n_max > 0 ? h->n_max : 1), s) !=
                cudaSuccess ||
            cudaMemsetAsync(h->pcount[0], 0, (size_t)h->U * sizeof(int), s) != cudaSuccess ||
            cudaMemsetAsync(h->pcount[1], 0, (size_t)h->U * sizeof(int), s) != cudaSuccess)
            return ISKV_ERR_CUDA;
    }
    if (cudaMemsetAsync(h->stats, 0, 4 * sizeof(unsigned long long),
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ISKV_ERR_CUDA;
    return ISKV_OK;
}

int iskv_fold_stats(iskv_handle *h, iskv_stream_t stream, int *max_sweeps_out,
                    long long *total_sweeps_out, long long *cores_out) {
    if (!h) return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    unsigned long long v[4] = {0, 0, 0, 0};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (join_all(h, s) != ISKV_OK) return ISKV_ERR_CUDA;
    if (cudaMemcpyAsync(v, h->stats, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ISKV_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ISKV_ERR_CUDA;
    if (max_sweeps_out) *max_sweeps_out = (int)v[0];
    if (total_sweeps_out) *total_sweeps_out = (long long)v[1];
    if (cores_out) *cores_out = (long long)v[2];
    return ISKV_OK;
}

int iskv_launch_count(const iskv_handle *h, long long *count_out) {
    if (!h || !count_out) return ISKV_ERR_INVALID_ARG;
    *count_out = h->launches;
    return ISKV_OK;
}

int iskv_num_tokens(const iskv_handle *h, int layer, long long *t_out) {
    if (!h || !t_out || !valid_layer(h, layer)) return ISKV_ERR_INVALID_ARG;
    *t_out = h->t[layer];
    return ISKV_OK;
}

int iskv_storage_bytes(const iskv_handle *h, int layer, long long *bytes_out) {
    if (!h || !bytes_out || !valid_layer(h, layer)) return ISKV_ERR_INVALID_ARG;
    const long long n = h->nc[layer], e = h->t[layer] - n;
    // factor units of the layer and the length d of their rows
    const long long fu = h->CL, d = h->joint ? (long long)h->cfg.n_kv_heads * D : D;
    long long f = 0;
    for (int x = 0; x < 2; ++x)
        f += (long long)h->kcur[x][layer] * ((long long)h->csz * n + 4LL * (d + 1));
    *bytes_out = fu * f + (long long)h->UL * (long long)h->esz * D * 2LL * e;
    return ISKV_OK;
}

int iskv_sync_status(iskv_handle *h, iskv_stream_t stream) {
    if (!h) return ISKV_ERR_INVALID_ARG;
    DeviceGuard g(h->device);
    int st = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (join_all(h, s) != ISKV_OK) return ISKV_ERR_CUDA;
    if (cudaMemcpyAsync(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ISKV_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ISKV_ERR_CUDA;
    return st;
}

}  // extern "C"
