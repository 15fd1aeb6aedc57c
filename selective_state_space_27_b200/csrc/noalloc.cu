// mamba_scan_fwd_noalloc: the selective scan forward for callers that cannot
// allocate device memory.
//
// mamba_scan_fwd asks its caller for a workspace whenever the sequence is
// split into segments (the multi-block carry). Some callers have no way to
// provide one: a plugin living inside a host application that owns every
// device allocation and hands the plugin nothing but its input and output
// buffers, or a latency-critical path where cudaMalloc is not allowed because
// it can synchronise the whole device. This entry point serves them: the
// carry workspace lives in a fixed, file-scope device array of kScratchBytes
// that every GPU loading this library holds until the process exits.
//
// The host-side name g_noalloc_scratch is only a stand-in for the device
// array; its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device. That first call should therefore come before any stream
// capture. All calls on a device share the one array and the array keeps
// whatever the previous call left in it: the kernels write every entry they
// later read, so nothing needs clearing, but two calls whose kernels overlap
// on the GPU (different streams, no ordering between them) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "launch.h"
#include "mambascan.h"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(MS_NOALLOC_SCRATCH_BYTES);
static_assert(kScratchBytes % 256 == 0, "scratch size must be a multiple of 256 bytes");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {nullptr};
int g_sms[kMaxDevices] = {0};
std::mutex g_mu;

template <typename... Args>
ms_status fail(ms_status st, const char *fmt, Args... args) {
    ms::record_error(fmt, args...);
    return st;
}

// Device address of the scratch array and the SM count of the current
// device, looked up on the first call made on that device.
ms_status device_setup(void **scratch, int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MS_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(MS_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr)
            return fail(MS_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(MS_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        g_sms[dev] = n;
        g_scratch_addr[dev] = ptr;
    }
    *scratch = g_scratch_addr[dev];
    *sms = g_sms[dev];
    return MS_OK;
}

}  // namespace

static ms_status noalloc_call(const ms_scan_args *args, void *stream) {
    // Validate exactly as mamba_scan_fwd does (the message, if any, is already recorded).
    size_t need = 0;
    ms_status st = mamba_scan_workspace_size(args, &need);
    if (st != MS_OK) return st;
    if (need > kScratchBytes)
        return fail(MS_ERR_WORKSPACE,
                    "this call needs %zu bytes of carry scratch; the built-in array holds %zu "
                    "(use mamba_scan_fwd with a caller-allocated workspace)",
                    need, kScratchBytes);
    void *scratch = nullptr;
    int sms = 0;
    st = device_setup(&scratch, &sms);
    if (st != MS_OK) return st;

    ms::ScanParams p{};
    p.batch = args->batch; p.dim = args->dim; p.dstate = args->dstate; p.seqlen = args->seqlen;
    p.u = args->u; p.u_sb = args->u_batch_stride; p.u_sd = args->u_dim_stride;
    p.delta = args->delta; p.dl_sb = args->delta_batch_stride; p.dl_sd = args->delta_dim_stride;
    p.B = args->B; p.B_sb = args->B_batch_stride; p.B_sn = args->B_state_stride;
    p.C = args->C; p.C_sb = args->C_batch_stride; p.C_sn = args->C_state_stride;
    p.z = args->z; p.z_sb = args->z_batch_stride; p.z_sd = args->z_dim_stride;
    p.y = args->y; p.y_sb = args->y_batch_stride; p.y_sd = args->y_dim_stride;
    p.A = args->A; p.D = args->D; p.delta_bias = args->delta_bias;
    p.h0 = args->initial_state; p.hT = args->final_state;
    p.softplus = args->delta_softplus ? 1 : 0;
    const ms::ScanPlan plan = ms::plan_scan(p, args->in_dtype, args->force_segments, sms);
    ms::bind_workspace(p, plan, scratch);
    const cudaError_t e = ms::launch_scan(p, plan, args->in_dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(MS_ERR_CUDA, "scan kernel launch: %s", cudaGetErrorString(e));
    return MS_OK;
}

extern "C" ms_status mamba_scan_fwd_noalloc(const ms_scan_args *args, void *stream) {
    nvtxRangePushA("mamba_scan_fwd_noalloc");
    const ms_status st = noalloc_call(args, stream);
    nvtxRangePop();
    return st;
}
