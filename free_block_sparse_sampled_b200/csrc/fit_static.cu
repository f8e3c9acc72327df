// sparsepr_probe_fit_static: the probe fit with its scratch in a static
// device array instead of a caller workspace.
//
// Who needs it: a caller that already holds the partition and routing
// results (and the probe outputs) but may not allocate device memory at the
// point where it fits, e.g. a host framework that has handed all free HBM to
// its own caching allocator, or a latency-critical loop that must not pay
// the device-wide synchronisation cudaMalloc/cudaFree imply.  The fit's
// scratch (fp64 statistics, Gram matrices and right-hand sides) is a few
// MiB, so it can live in one static array that every GPU loading the library
// holds until the process exits.
//
// The kernels are the ones sparsepr_probe_fit launches; only the scratch
// addresses differ.  The array is shared by every call on a device and keeps
// the previous call's contents; the only word that must start at zero (the
// device status) is cleared at the start of each call.  Calls whose work
// overlaps on the GPU (other streams, other host threads) race on it.
#include <mutex>

#include "common.cuh"
#include "internal.h"

// Every device that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_fit_scratch[SPARSEPR_FIT_STATIC_SCRATCH_BYTES];

namespace spr {

namespace {

constexpr size_t kStaticScratchBytes = SPARSEPR_FIT_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

size_t up256(size_t b) { return (b + 255) / 256 * 256; }

// Scratch layout: status word, psum[BH], fstat[BH,3,d], G[BH,d,d], rhs[BH,d,d].
struct StaticLayout {
    size_t o_status, o_psum, o_fstat, o_G, o_rhs, total;
};

StaticLayout static_layout(size_t BH, size_t d) {
    StaticLayout L;
    size_t c = 0;
    L.o_status = c; c += up256(sizeof(DevStatus));
    L.o_psum = c;   c += up256(BH * sizeof(int32_t));
    L.o_fstat = c;  c += up256(BH * 3 * d * sizeof(double));
    L.o_G = c;      c += up256(BH * d * d * sizeof(double));
    L.o_rhs = c;    c += up256(BH * d * d * sizeof(double));
    L.total = c;
    return L;
}

// Device address of the scratch array on the current device, looked up once
// per device.  The lookup may load the module, so the first call on a device
// should come before any stream capture.  The cached address belongs to the
// context current at that lookup and is not refreshed: it does not survive a
// cudaDeviceReset of the device.
sparsepr_status scratch_address(void** out) {
    int dev = 0;
    sparsepr_status s = cuda_status(cudaGetDevice(&dev));
    if (s != SPARSEPR_OK) return s;
    if (dev < 0 || dev >= kMaxDevices) {
        snprintf(last_error_buffer(), 256, "sparsepr_probe_fit_static: device %d beyond the %d supported", dev,
                 kMaxDevices);
        return SPARSEPR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        s = cuda_status(cudaGetSymbolAddress(&ptr, g_fit_scratch));
        if (s != SPARSEPR_OK) return s;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return SPARSEPR_OK;
}

}  // namespace

}  // namespace spr

using namespace spr;

extern "C" {

sparsepr_status sparsepr_probe_fit_static(const sparsepr_params* p, const sparsepr_partition_out* part,
                                          const sparsepr_route_out* route, const float* probe_sparse,
                                          const float* probe_dense, const sparsepr_fit_out* fit,
                                          int32_t* device_status, void* stream) {
    if (p == nullptr) return SPARSEPR_INVALID_ARG;
    const sparsepr_status v = sparsepr_validate(p);
    if (v != SPARSEPR_OK) return v;
    if (p->residual_rank > 0) {
        snprintf(last_error_buffer(), 256, "sparsepr_probe_fit_static: rank truncation needs a workspace");
        return SPARSEPR_UNSUPPORTED;
    }
    Plan pl;
    if (!make_plan(*p, pl)) return SPARSEPR_INVALID_ARG;
    if (!part || !part->q_offsets || !part->n_groups || !route || !route->probe_alloc ||
        (pl.Mp > 0 && (!route->probe_group || !probe_sparse || !probe_dense)) || !fit || !fit->B || !fit->mu_x ||
        !fit->sigma || !fit->mu_r)
        return SPARSEPR_INVALID_ARG;
    const StaticLayout L = static_layout((size_t)pl.BH, (size_t)pl.d);
    if (L.total > kStaticScratchBytes) {
        snprintf(last_error_buffer(), 256,
                 "sparsepr_probe_fit_static: B*H=%d, d=%d needs %zu bytes of scratch; the static limit is %zu",
                 pl.BH, pl.d, L.total, kStaticScratchBytes);
        return SPARSEPR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    sparsepr_status s = scratch_address(&scratch);
    if (s != SPARSEPR_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the previous call's status word must not leak into this one
    s = cuda_status(cudaMemsetAsync(at<void>(scratch, L.o_status), 0, sizeof(int32_t) * 2, st));
    if (s != SPARSEPR_OK) return s;
    // run_fit reads its scratch through the plan's offsets: point them into the array
    Plan sp = pl;
    sp.o_status = L.o_status;
    sp.o_psum = L.o_psum;
    sp.o_fstat = L.o_fstat;
    sp.o_G = L.o_G;
    sp.o_rhs = L.o_rhs;
    s = run_fit(*p, sp, *part, *route, probe_sparse, probe_dense, *fit, scratch, st);
    if (s != SPARSEPR_OK) return s;
    if (device_status != nullptr)
        s = cuda_status(cudaMemcpyAsync(device_status, at<void>(scratch, L.o_status), sizeof(int32_t),
                                        cudaMemcpyDeviceToDevice, st));
    return s;
}

}  // extern "C"
