// hs2_sparse_attn_static: the sparse-attention layer (KV Reuse over caller indices) with its
// scratch in a fixed device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory when they need this call: a serving engine that
// hands out all device memory from its own fixed pools and forbids allocation on the request
// path, a plugin loaded into a host program that owns the device memory, or code on a latency
// budget that cannot afford an allocation (or a workspace query) per call.  For them the
// scratch this layer needs -- its split partials and per-row counters -- lives in one
// file-scope device array, HS2_STATIC_SCRATCH_BYTES large, that every GPU which loads the
// library holds until the process exits.
//
// The kernels are the ones hs2_sparse_attn launches; only where their scratch lives differs.
// Host code cannot use the array's name as a device address (it stands for a host-side shadow),
// so the first call on each device looks the address up with cudaGetSymbolAddress while that
// device is current, and later calls reuse it.  The cached address belongs to the device context
// it was looked up in: after cudaDeviceReset the array is reallocated and the cache is stale.
#include <mutex>

#include "hs2_internal.h"

namespace hs2 {
namespace {

constexpr size_t kStaticScratch = HS2_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratch];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
hs2_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HS2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return HS2_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HS2_OK;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" hs2_status hs2_sparse_attn_static(const hs2_dims* dims, const void* Q_sparse, const void* K,
                                             const void* V, const int32_t* pos, const int32_t* idx,
                                             const int32_t* cnt, void* O_sparse, float* LSE_sparse,
                                             void* stream) {
    Plan p;
    hs2_status why;
    if (!make_plan(dims, &p, &why)) return why;
    auto a16 = [](const void* q) { return q && (reinterpret_cast<uintptr_t>(q) % 16) == 0; };
    auto a4 = [](const void* q) { return q && (reinterpret_cast<uintptr_t>(q) % 4) == 0; };
    const bool idx_ok = (p.k + p.W == 0 && !idx) || a4(idx);
    if (!a16(Q_sparse) || !a16(K) || !a16(V) || !a4(pos) || !idx_ok || !a4(cnt) || !a16(O_sparse) ||
        !a4(LSE_sparse))
        return HS2_ERR_INVALID_ARG;

    // layout inside the fixed scratch: status word | per-row counters | split partials
    const size_t off_meta = 256;
    const size_t meta_end = up256(off_meta + static_cast<size_t>(p.rows_kv) * kMetaInts * 4);
    const size_t off_ml = meta_end;
    const size_t off_acc = up256(off_ml + static_cast<size_t>(p.S4) * p.rows_q * 8);
    const size_t need = up256(off_acc + static_cast<size_t>(p.S4) * p.rows_q * p.d * 4);
    if (need > kStaticScratch) return HS2_ERR_WORKSPACE;  // too large for the built-in scratch

    void* scratch = nullptr;
    const hs2_status s = scratch_address(&scratch);
    if (s != HS2_OK) return s;
    uint8_t* base = static_cast<uint8_t*>(scratch);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // the array keeps the previous call's contents: clear the status word and the counters
    trace_call_begin(st);
    if (launch_init(base, meta_end, st) != cudaSuccess) return HS2_ERR_CUDA;
    SparseArgs sa{};
    sa.Q = static_cast<const uint16_t*>(Q_sparse);
    sa.K = static_cast<const uint16_t*>(K);
    sa.V = static_cast<const uint16_t*>(V);
    sa.pos = pos;
    sa.idx = idx;
    sa.cnt = cnt;
    sa.B = p.B; sa.Hq = p.Hq; sa.Hkv = p.Hkv; sa.T = p.T; sa.N = p.N; sa.G = p.G; sa.kw = p.k + p.W;
    sa.C4 = p.C4; sa.S4 = p.S4;
    sa.kv.page_shift = -1;  // contiguous bf16 cache
    sa.scale_log2 = kLog2e / sqrtf(static_cast<float>(p.d));
    sa.part_ml = reinterpret_cast<float2*>(base + off_ml);
    sa.part_acc = reinterpret_cast<float*>(base + off_acc);
    sa.meta = reinterpret_cast<int*>(base + off_meta);
    sa.O = static_cast<uint16_t*>(O_sparse);
    sa.LSE = LSE_sparse;
    sa.status = reinterpret_cast<unsigned*>(base);
    return launch_sparse_attn(p, sa, st) == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}
