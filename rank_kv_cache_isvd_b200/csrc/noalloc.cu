// Decode attention over caller-owned buffers that allocates nothing: the split partials live in a
// fixed file-scope device array instead of handle-owned memory (see iskv_decode_attn_noalloc in
// include/iskv.h for who needs this and the limits). The kernels are the CUDA-core decode kernels
// that iskv_decode_attn() uses when the tensor-core path does not apply.
#include <math.h>
#include <string.h>

#include <mutex>

#include "iskv_internal.cuh"

using namespace iskv;

namespace {

// Scratch for split partials of iskv_decode_attn_noalloc(); every GPU that loads the library holds
// it until exit. Shared by all calls: overlapping calls on the GPU race.
static __device__ __align__(256) float g_noalloc_scratch[ISKV_NOALLOC_SCRATCH_FLOATS];

// Same device limit as the per-device function attributes of the decode launchers (64).
constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once per device (with the
// device current). In host code the array's name is only a host-side stand-in, never a device
// address, so it is never passed to a kernel directly.
float *scratch_for_current_device(int *err) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *err = ISKV_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            *err = ISKV_ERR_CUDA;
            return nullptr;
        }
        g_scratch_addr[dev] = static_cast<float *>(p);
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" int iskv_decode_attn_noalloc(const iskv_decode_view *v, const float *q, float *out,
                                        iskv_stream_t stream) {
    if (!v || !q || !out) return ISKV_ERR_INVALID_ARG;
    if (v->head_dim != D || v->batch < 1 || v->n_kv_heads < 1 || v->n_q_heads < v->n_kv_heads ||
        v->n_q_heads % v->n_kv_heads != 0 || v->n_q_heads / v->n_kv_heads > GMAX ||
        v->rank_k < 1 || v->rank_k > D || v->rank_v < 1 || v->rank_v > D || v->t < 1 ||
        v->n_c < 0 || v->n_c > v->t || v->n_c > v->n_max || v->ring_rows < 1 ||
        v->t - v->n_c > v->ring_rows || (v->kv_dtype != ISKV_BF16 && v->kv_dtype != ISKV_F32) ||
        !v->ring_k || !v->ring_v)
        return ISKV_ERR_INVALID_ARG;
    if (v->n_c > 0 && (v->k_k < 1 || v->k_k > v->rank_k || v->k_v < 1 || v->k_v > v->rank_v ||
                       !v->coords_k || !v->coords_v || !v->basis_k || !v->basis_v))
        return ISKV_ERR_INVALID_ARG;
    const int units = v->batch * v->n_kv_heads;
    const int G = v->n_q_heads / v->n_kv_heads;
    // the window splits alone (one per 128 exact rows) are a lower bound on the split count that
    // needs no device query: requests that cannot fit are refused before any CUDA call
    const long long wsplits = (v->t - v->n_c + DEC_TILE - 1) / DEC_TILE + (v->n_c > 0 ? 1 : 0);
    if ((long long)units * wsplits * G * (2 + D) > ISKV_NOALLOC_SCRATCH_FLOATS)
        return ISKV_ERR_CAPACITY;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ISKV_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms < 1) {
        cudaGetLastError();
        return ISKV_ERR_CUDA;
    }

    DecodeArgs da;
    memset(&da, 0, sizeof(da));
    const long long ctiles = (v->n_c + DEC_TILE - 1) / DEC_TILE;
    const long long target = 2LL * sms;
    long long tps = (ctiles * units + target - 1) / target;
    if (tps < 1) tps = 1;
    da.split_rows = (int)(tps * DEC_TILE);
    da.n_split_c = (int)((ctiles + tps - 1) / tps);
    da.n_split = da.n_split_c + (int)((v->t - v->n_c + DEC_TILE - 1) / DEC_TILE);
    da.max_splits = da.n_split;
    const long long need = (long long)units * da.n_split * G * (2 + D);
    if (need > ISKV_NOALLOC_SCRATCH_FLOATS) return ISKV_ERR_CAPACITY;
    int err = ISKV_OK;
    float *scratch = scratch_for_current_device(&err);
    if (!scratch) return err;

    da.coords[0] = v->coords_k;
    da.coords[1] = v->coords_v;
    da.basis[0] = v->basis_k;
    da.basis[1] = v->basis_v;
    da.ring[0] = v->ring_k;
    da.ring[1] = v->ring_v;
    da.rope_cs = reinterpret_cast<const float2 *>(v->rope_cs);
    da.q = q;
    da.out = out;
    da.ws = scratch;
    da.r[0] = v->rank_k;
    da.r[1] = v->rank_v;
    da.k[0] = v->n_c > 0 ? v->k_k : 0;
    da.k[1] = v->n_c > 0 ? v->k_v : 0;
    da.n_c = v->n_c;
    da.t = v->t;
    da.n_max = v->n_max;
    da.R = v->ring_rows;
    da.H = v->n_kv_heads;
    da.G = G;
    da.kv_dtype = v->kv_dtype;
    da.scale = 1.0f / sqrtf((float)D);
    da.new_pos = -1;
    return launch_decode(da, units, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? ISKV_OK
               : ISKV_ERR_CUDA;
}
