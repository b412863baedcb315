// kda_noalloc.cu -- kda_chunk_fwd_noalloc: the chunk forward with no allocation.
//
// Some callers cannot call cudaMalloc: code that must not synchronise the
// device (cudaMalloc may), loops that forbid allocation once they are running,
// and host applications that own the whole device pool and hand a component
// no allocator.  For them this entry point runs the FP32 two-phase chunk path
// with its scratch in a fixed file-scope device array instead of a
// caller-supplied workspace.
//
// The array is KDA_NOALLOC_SCRATCH_BYTES (32 MiB) and lives on every GPU that
// loads the library until the process exits.  Its device address is looked up
// once per device (cudaGetSymbolAddress, on the first call made with that
// device current) and cached; that first call should therefore come before any
// stream capture.  Every call shares the array: calls whose work overlaps on
// the GPU (different streams, or different host threads on one device) race.
// Each call writes every scratch element it later reads, so nothing needs to
// start at zero and the previous call's leftovers are never used.  The cached
// address belongs to the device's primary context: after cudaDeviceReset (or any
// other teardown of that context) this entry point must not be called again in
// the same process.
#include <mutex>
#include <string.h>

#include "../../include/kda.h"
#include "kda_internal.h"
#include "kda_checks.h"

using namespace kda;

static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array for the current device (NULL on error).
void *scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
}  // namespace

extern "C" int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                                     const void *beta, const float *S0, void *out, float *S_T,
                                     int B, int T, int H, int dk, int dv, const kda_opts *opts,
                                     cudaStream_t stream) {
    kda_opts o;
    memset(&o, 0, sizeof(o));
    o.dtype = KDA_BF16;
    o.flags = KDA_QK_L2NORM;
    o.scale = 1.0f;
    if (opts) o = *opts;
    // the same argument rules as kda_chunk_fwd; the flags that only choose among its paths
    // (KDA_FUSED, KDA_SPLIT, KDA_UNBOUNDED_DECAY, KDA_GATE_SOFTPLUS) are accepted and have no
    // effect here: this entry point always runs the exact-FP32 path, which takes any g <= 0
    int st = check_opts(o);
    if (st != KDA_OK) return st;
    if ((st = check_dims(B, T, H, dk, dv)) != KDA_OK) return st;
    if (B == 0 || H == 0) return KDA_OK;
    if (T == 0) {
        if (!aligned16(S0) || !aligned16(S_T)) return KDA_ERR_ALIGN;
        if (!S_T) return KDA_OK;
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(S_T, 0, bytes, stream);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    // the fixed scratch bounds the sizes this entry point accepts
    const size_t need = chunk_ref_workspace_bytes(B, T, H, dk, dv);
    if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
    if (!q || !k || !v || !g || !beta || !out) return KDA_ERR_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, out, S_T};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGN;
    void *scratch = scratch_for_current_device();
    if (!scratch) return KDA_ERR_CUDA;

    ChunkArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
    const Elt t = o.dtype == KDA_BF16 ? Elt::BF16 : Elt::F32;
    a.t_qkv = a.t_g = a.t_beta = a.t_out = t;
    a.S0 = S0; a.out = out; a.S_T = S_T;
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
    a.fl.l2norm = (o.flags & KDA_QK_L2NORM) ? 1 : 0;
    a.fl.complex_gate = (o.flags & KDA_COMPLEX) ? 1 : 0;
    a.fl.scale = o.scale;
    a.workspace = scratch;
    a.workspace_bytes = KDA_NOALLOC_SCRATCH_BYTES;
    int launches = 0;
    a.launch_idx = &launches;
    a.events = o.events; a.n_events = o.n_events;
    cudaError_t e = launch_chunk_ref(a, stream);
    if (e == cudaSuccess && o.events && launches < o.n_events) cudaEventRecord(o.events[launches], stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
