// C ABI of the selective-scan library: argument validation, launch planning
// and dispatch. Declarations and the contract are in include/mambascan.h.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "launch.h"
#include "mambascan.h"

namespace {

// An NVTX range named after the entry point for the duration of the call, so
// that profilers (ncu --nvtx, nsys) can attribute the launches; without a
// profiler attached the push and pop return at once.
struct CallRange {
    explicit CallRange(const char *name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;
};

thread_local char g_last_error[512] = "";

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}

ms_status invalid(const char *what) {
    set_error("invalid argument: %s", what);
    return MS_ERR_INVALID_ARG;
}

ms_status cuda_fail(cudaError_t e, const char *where) {
    set_error("%s: %s", where, cudaGetErrorString(e));
    return MS_ERR_CUDA;
}

// Number of SMs of the current device, cached per device.
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
std::mutex g_sms_mu;

ms_status device_sms(int *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev >= 0 && dev < kMaxDevices) {
        std::lock_guard<std::mutex> lk(g_sms_mu);
        if (g_sms[dev] == 0) {
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
            g_sms[dev] = sms;
        }
        *out = g_sms[dev];
        return MS_OK;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    *out = sms;
    return MS_OK;
}

bool elem_aligned(const void *ptr, int eb) {
    return (reinterpret_cast<uintptr_t>(ptr) % static_cast<uintptr_t>(eb)) == 0;
}

ms_status check_scan(const ms_scan_args *a) {
    if (!a) return invalid("args is NULL");
    if (a->batch <= 0 || a->dim <= 0 || a->dstate <= 0 || a->seqlen <= 0)
        return invalid("batch, dim, dstate and seqlen must be positive");
    if (a->in_dtype != MS_F32 && a->in_dtype != MS_BF16) return invalid("in_dtype");
    if (a->reserved != 0) return invalid("reserved must be 0");
    if (a->force_segments < 0) return invalid("force_segments must be >= 0");
    if (!a->u || !a->delta || !a->B || !a->C || !a->A || !a->y)
        return invalid("u, delta, B, C, A and y are required");
    if (a->u_batch_stride < 0 || a->u_dim_stride < 0 || a->delta_batch_stride < 0 ||
        a->delta_dim_stride < 0 || a->B_batch_stride < 0 || a->B_state_stride < 0 ||
        a->C_batch_stride < 0 || a->C_state_stride < 0 || a->y_batch_stride < 0 ||
        a->y_dim_stride < 0 || (a->z && (a->z_batch_stride < 0 || a->z_dim_stride < 0)))
        return invalid("strides must be non-negative");
    if (a->dstate > MS_MAX_DSTATE) {
        set_error("dstate %lld exceeds the supported maximum %d", static_cast<long long>(a->dstate),
                  MS_MAX_DSTATE);
        return MS_ERR_UNSUPPORTED;
    }
    if (a->batch > 65535) {
        set_error("batch %lld exceeds 65535", static_cast<long long>(a->batch));
        return MS_ERR_UNSUPPORTED;
    }
    const int eb = a->in_dtype == MS_F32 ? 4 : 2;
    if (!elem_aligned(a->u, eb) || !elem_aligned(a->delta, eb) || !elem_aligned(a->B, eb) ||
        !elem_aligned(a->C, eb) || !elem_aligned(a->y, eb) || (a->z && !elem_aligned(a->z, eb)) ||
        !elem_aligned(a->A, 4) || (a->D && !elem_aligned(a->D, 4)) ||
        (a->delta_bias && !elem_aligned(a->delta_bias, 4)) ||
        (a->initial_state && !elem_aligned(a->initial_state, 4)) ||
        (a->final_state && !elem_aligned(a->final_state, 4))) {
        set_error("a pointer is not aligned to its element size");
        return MS_ERR_ALIGNMENT;
    }
    return MS_OK;
}

ms::ScanParams to_params(const ms_scan_args *a) {
    ms::ScanParams p{};
    p.batch = a->batch; p.dim = a->dim; p.dstate = a->dstate; p.seqlen = a->seqlen;
    p.u = a->u; p.u_sb = a->u_batch_stride; p.u_sd = a->u_dim_stride;
    p.delta = a->delta; p.dl_sb = a->delta_batch_stride; p.dl_sd = a->delta_dim_stride;
    p.B = a->B; p.B_sb = a->B_batch_stride; p.B_sn = a->B_state_stride;
    p.C = a->C; p.C_sb = a->C_batch_stride; p.C_sn = a->C_state_stride;
    p.z = a->z; p.z_sb = a->z_batch_stride; p.z_sd = a->z_dim_stride;
    p.y = a->y; p.y_sb = a->y_batch_stride; p.y_sd = a->y_dim_stride;
    p.A = a->A; p.D = a->D; p.delta_bias = a->delta_bias;
    p.h0 = a->initial_state; p.hT = a->final_state;
    p.softplus = a->delta_softplus ? 1 : 0;
    return p;
}

ms_status check_conv(const ms_conv1d_args *c) {
    if (!c) return invalid("conv is NULL");
    if (!c->weight) return invalid("conv weight is required");
    if (c->silu != 0 && c->silu != 1) return invalid("conv silu must be 0 or 1");
    if (c->width < 1) return invalid("conv width must be >= 1");
    if (c->width > MS_MAX_CONV_WIDTH) {
        set_error("conv width %d exceeds the supported maximum %d", c->width, MS_MAX_CONV_WIDTH);
        return MS_ERR_UNSUPPORTED;
    }
    if (!elem_aligned(c->weight, 4) || (c->bias && !elem_aligned(c->bias, 4))) {
        set_error("conv weight or bias is not aligned to 4 bytes");
        return MS_ERR_ALIGNMENT;
    }
    return MS_OK;
}

// Validate a decode call and fill its kernel parameters.
ms_status update_params(const ms_update_args *a, ms::UpdateParams *p) {
    if (!a) return invalid("args is NULL");
    if (a->batch <= 0 || a->dim <= 0 || a->dstate <= 0)
        return invalid("batch, dim and dstate must be positive");
    if (a->in_dtype != MS_F32 && a->in_dtype != MS_BF16) return invalid("in_dtype");
    if (!a->state || !a->x || !a->delta || !a->B || !a->C || !a->A || !a->y)
        return invalid("state, x, delta, B, C, A and y are required");
    if (a->state_batch_stride < 0 || a->state_dim_stride < 0 || a->x_batch_stride < 0 ||
        a->delta_batch_stride < 0 || a->B_batch_stride < 0 || a->C_batch_stride < 0 ||
        a->y_batch_stride < 0 || (a->z && a->z_batch_stride < 0))
        return invalid("strides must be non-negative");
    if (a->dstate > MS_MAX_DSTATE) {
        set_error("dstate %lld exceeds the supported maximum %d", static_cast<long long>(a->dstate),
                  MS_MAX_DSTATE);
        return MS_ERR_UNSUPPORTED;
    }
    if (a->batch > 65535) {
        set_error("batch %lld exceeds 65535", static_cast<long long>(a->batch));
        return MS_ERR_UNSUPPORTED;
    }
    const int eb = a->in_dtype == MS_F32 ? 4 : 2;
    if (!elem_aligned(a->state, 4) || !elem_aligned(a->x, eb) || !elem_aligned(a->delta, eb) ||
        !elem_aligned(a->B, eb) || !elem_aligned(a->C, eb) || !elem_aligned(a->y, eb) ||
        (a->z && !elem_aligned(a->z, eb)) || !elem_aligned(a->A, 4) ||
        (a->D && !elem_aligned(a->D, 4)) || (a->delta_bias && !elem_aligned(a->delta_bias, 4))) {
        set_error("a pointer is not aligned to its element size");
        return MS_ERR_ALIGNMENT;
    }
    *p = ms::UpdateParams{};
    p->batch = a->batch; p->dim = a->dim; p->dstate = a->dstate;
    p->state = a->state; p->s_sb = a->state_batch_stride; p->s_sd = a->state_dim_stride;
    p->x = a->x; p->x_sb = a->x_batch_stride;
    p->delta = a->delta; p->dl_sb = a->delta_batch_stride;
    p->B = a->B; p->B_sb = a->B_batch_stride;
    p->C = a->C; p->C_sb = a->C_batch_stride;
    p->z = a->z; p->z_sb = a->z_batch_stride;
    p->y = a->y; p->y_sb = a->y_batch_stride;
    p->A = a->A; p->D = a->D; p->delta_bias = a->delta_bias;
    p->softplus = a->delta_softplus ? 1 : 0;
    return MS_OK;
}

ms_status run_plan(ms::ScanParams p, const ms::ScanPlan &plan, int in_dtype, void *workspace,
                   size_t workspace_bytes, void *stream) {
    if (plan.ws_bytes > 0) {
        if (!workspace || workspace_bytes < plan.ws_bytes) {
            set_error("workspace of %zu bytes needed, %zu given", plan.ws_bytes,
                      workspace ? workspace_bytes : static_cast<size_t>(0));
            return MS_ERR_WORKSPACE;
        }
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
            set_error("workspace must be 256-byte aligned");
            return MS_ERR_ALIGNMENT;
        }
    }
    ms::bind_workspace(p, plan, workspace);
    const cudaError_t e = ms::launch_scan(p, plan, in_dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
    return MS_OK;
}

}  // namespace

namespace ms {
void record_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}
}  // namespace ms

extern "C" {

const char *mamba_status_string(int status) {
    switch (status) {
        case MS_OK: return "MS_OK";
        case MS_ERR_INVALID_ARG: return "MS_ERR_INVALID_ARG";
        case MS_ERR_UNSUPPORTED: return "MS_ERR_UNSUPPORTED";
        case MS_ERR_ALIGNMENT: return "MS_ERR_ALIGNMENT";
        case MS_ERR_CUDA: return "MS_ERR_CUDA";
        case MS_ERR_TIMEOUT: return "MS_ERR_TIMEOUT";
        case MS_ERR_WORKSPACE: return "MS_ERR_WORKSPACE";
        default: return "MS_UNKNOWN_STATUS";
    }
}

const char *mamba_last_error(void) { return g_last_error; }

int mamba_abi_version(void) { return MAMBASCAN_ABI_VERSION; }

ms_status mamba_scan_workspace_size(const ms_scan_args *args, size_t *bytes) {
    if (!bytes) return invalid("bytes is NULL");
    *bytes = 0;
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    const ms::ScanParams p = to_params(args);
    *bytes = ms::plan_scan(p, args->in_dtype, args->force_segments, sms).ws_bytes;
    return MS_OK;
}

ms_status mamba_scan_fwd(const ms_scan_args *args, void *workspace, size_t workspace_bytes,
                         void *stream) {
    const CallRange range("mamba_scan_fwd");
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    const ms::ScanParams p = to_params(args);
    const ms::ScanPlan plan = ms::plan_scan(p, args->in_dtype, args->force_segments, sms);
    return run_plan(p, plan, args->in_dtype, workspace, workspace_bytes, stream);
}

int mamba_scan_num_configs(void) { return ms::scan_num_configs(); }

ms_status mamba_scan_config_info(int config, int *lanes, int *states_per_pass, int *max_warps) {
    if (!ms::scan_config_info(config, lanes, states_per_pass, max_warps)) return invalid("unknown config");
    return MS_OK;
}

ms_status mamba_scan_config_kind(int config, int *kind) {
    if (!kind) return invalid("kind is NULL");
    *kind = ms::scan_config_kind(config);
    if (*kind < 0) return invalid("unknown config");
    return MS_OK;
}

ms_status mamba_scan_plan_query(const ms_scan_args *args, ms_scan_plan *plan) {
    if (!plan) return invalid("plan is NULL");
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    const ms::ScanPlan pl = ms::plan_scan(to_params(args), args->in_dtype, args->force_segments, sms);
    plan->config = pl.config;
    plan->warps_per_cta = pl.warps;
    plan->segments = pl.nseg;
    plan->lanes = pl.lg;
    plan->segment_len = pl.seg_len;
    plan->workspace_bytes = pl.ws_bytes;
    plan->ctas = pl.ctas;
    plan->reserved = 0;
    return MS_OK;
}

ms_status mamba_scan_plan_workspace_size(const ms_scan_args *args, const ms_scan_plan *plan, size_t *bytes) {
    if (!bytes) return invalid("bytes is NULL");
    *bytes = 0;
    if (!plan) return invalid("plan is NULL");
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    ms::ScanPlan pl{};
    if (!ms::make_plan(to_params(args), args->in_dtype, plan->config, plan->warps_per_cta, plan->segments,
                       plan->ctas, sms, &pl)) {
        set_error("plan (config %d, %d warps, %d segments, %d CTAs) cannot run these arguments", plan->config,
                  plan->warps_per_cta, plan->segments, plan->ctas);
        return MS_ERR_UNSUPPORTED;
    }
    *bytes = pl.ws_bytes;
    return MS_OK;
}

ms_status mamba_scan_fwd_with_plan(const ms_scan_args *args, const ms_scan_plan *plan, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    const CallRange range("mamba_scan_fwd_with_plan");
    if (!plan) return invalid("plan is NULL");
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    const ms::ScanParams p = to_params(args);
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    ms::ScanPlan pl{};
    if (plan->reserved != 0 ||
        !ms::make_plan(p, args->in_dtype, plan->config, plan->warps_per_cta, plan->segments, plan->ctas, sms, &pl)) {
        set_error("plan (config %d, %d warps, %d segments, %d CTAs) cannot run these arguments", plan->config,
                  plan->warps_per_cta, plan->segments, plan->ctas);
        return MS_ERR_UNSUPPORTED;
    }
    return run_plan(p, pl, args->in_dtype, workspace, workspace_bytes, stream);
}

ms_status mamba_state_update(const ms_update_args *a, void *stream) {
    const CallRange range("mamba_state_update");
    ms::UpdateParams p;
    const ms_status st = update_params(a, &p);
    if (st != MS_OK) return st;
    const cudaError_t e = ms::launch_state_update(p, a->in_dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state update kernel launch");
    return MS_OK;
}

ms_status mamba_conv_state_update(const ms_update_args *a, const ms_conv1d_args *conv, void *conv_state,
                                  int64_t conv_state_batch_stride, int64_t conv_state_dim_stride,
                                  void *stream) {
    const CallRange range("mamba_conv_state_update");
    ms::UpdateParams p;
    ms_status st = update_params(a, &p);
    if (st != MS_OK) return st;
    st = check_conv(conv);
    if (st != MS_OK) return st;
    if (!conv_state) return invalid("conv_state is required");
    if (conv_state_batch_stride < 0 || conv_state_dim_stride < 0)
        return invalid("conv_state strides must be non-negative");
    if (!elem_aligned(conv_state, a->in_dtype == MS_F32 ? 4 : 2)) {
        set_error("conv_state is not aligned to its element size");
        return MS_ERR_ALIGNMENT;
    }
    p.conv_state = conv_state;
    p.cs_sb = conv_state_batch_stride;
    p.cs_sd = conv_state_dim_stride;
    p.conv_w = conv->weight;
    p.conv_b = conv->bias;
    p.conv_width = conv->width;
    p.conv_silu = conv->silu;
    const cudaError_t e = ms::launch_state_update(p, a->in_dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state update kernel launch");
    return MS_OK;
}

static ms_status conv_scan_impl(const ms_scan_args *args, const ms_conv1d_args *conv, const ms_scan_plan *plan,
                                void *workspace, size_t workspace_bytes, void *stream, bool with_workspace,
                                size_t *query) {
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    st = check_conv(conv);
    if (st != MS_OK) return st;
    if (args->force_segments > 1) {
        set_error("the convolution prologue runs in one segment (force_segments %d)", args->force_segments);
        return MS_ERR_UNSUPPORTED;
    }
    ms::ScanParams p = to_params(args);
    p.conv_w = conv->weight;
    p.conv_b = conv->bias;
    p.conv_width = conv->width;
    p.conv_silu = conv->silu;
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    ms::ScanPlan pl{};
    if (plan) {
        if ((!with_workspace && plan->ctas != 0) || plan->reserved != 0 ||
            !ms::make_plan(p, args->in_dtype, plan->config, plan->warps_per_cta, plan->segments, plan->ctas, sms,
                           &pl)) {
            set_error("plan (config %d, %d warps, %d segments, %d CTAs) cannot run the convolution prologue",
                      plan->config, plan->warps_per_cta, plan->segments, plan->ctas);
            return MS_ERR_UNSUPPORTED;
        }
    } else {
        pl = ms::plan_scan(p, args->in_dtype, 0, sms, with_workspace);
        if (pl.kind != 1) {
            set_error("no kernel configuration fuses the convolution prologue for these arguments");
            return MS_ERR_UNSUPPORTED;
        }
    }
    if (query) {
        *query = pl.ws_bytes;
        return MS_OK;
    }
    return run_plan(p, pl, args->in_dtype, workspace, workspace_bytes, stream);
}

ms_status mamba_conv_scan_fwd(const ms_scan_args *args, const ms_conv1d_args *conv, const ms_scan_plan *plan,
                              void *stream) {
    const CallRange range("mamba_conv_scan_fwd");
    return conv_scan_impl(args, conv, plan, nullptr, 0, stream, false, nullptr);
}

ms_status mamba_conv_scan_workspace_size(const ms_scan_args *args, const ms_conv1d_args *conv,
                                         const ms_scan_plan *plan, size_t *bytes) {
    if (!bytes) return invalid("bytes is NULL");
    *bytes = 0;
    return conv_scan_impl(args, conv, plan, nullptr, 0, nullptr, true, bytes);
}

ms_status mamba_conv_scan_fwd_ws(const ms_scan_args *args, const ms_conv1d_args *conv, const ms_scan_plan *plan,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    const CallRange range("mamba_conv_scan_fwd_ws");
    return conv_scan_impl(args, conv, plan, workspace, workspace_bytes, stream, true, nullptr);
}

static ms_status trap_scan_impl(const ms_scan_args *args, const void *lambda_raw, int64_t lambda_batch_stride,
                                int64_t lambda_dim_stride, const ms_scan_plan *plan, void *workspace,
                                size_t workspace_bytes, void *stream, bool with_workspace, size_t *query) {
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    if (!lambda_raw) return invalid("lambda_raw is required");
    if (lambda_batch_stride < 0 || lambda_dim_stride < 0) return invalid("lambda strides must be non-negative");
    if (!elem_aligned(lambda_raw, args->in_dtype == MS_F32 ? 4 : 2)) {
        set_error("lambda_raw is not aligned to its element size");
        return MS_ERR_ALIGNMENT;
    }
    if (args->force_segments > 1) {
        set_error("the trapezoidal rule runs in one segment (force_segments %d)", args->force_segments);
        return MS_ERR_UNSUPPORTED;
    }
    ms::ScanParams p = to_params(args);
    p.lambda_raw = lambda_raw;
    p.lm_sb = lambda_batch_stride;
    p.lm_sd = lambda_dim_stride;
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    ms::ScanPlan pl{};
    if (plan) {
        if ((!with_workspace && plan->ctas != 0) || plan->reserved != 0 ||
            !ms::make_plan(p, args->in_dtype, plan->config, plan->warps_per_cta, plan->segments, plan->ctas, sms,
                           &pl)) {
            set_error("plan (config %d, %d warps, %d segments, %d CTAs) cannot run the trapezoidal rule",
                      plan->config, plan->warps_per_cta, plan->segments, plan->ctas);
            return MS_ERR_UNSUPPORTED;
        }
    } else {
        pl = ms::plan_scan(p, args->in_dtype, 0, sms, with_workspace);
        if (pl.kind != 1) {
            set_error("no kernel configuration runs the trapezoidal rule for these arguments");
            return MS_ERR_UNSUPPORTED;
        }
    }
    if (query) {
        *query = pl.ws_bytes;
        return MS_OK;
    }
    return run_plan(p, pl, args->in_dtype, workspace, workspace_bytes, stream);
}

ms_status mamba_trap_scan_fwd(const ms_scan_args *args, const void *lambda_raw, int64_t lambda_batch_stride,
                              int64_t lambda_dim_stride, const ms_scan_plan *plan, void *stream) {
    const CallRange range("mamba_trap_scan_fwd");
    return trap_scan_impl(args, lambda_raw, lambda_batch_stride, lambda_dim_stride, plan, nullptr, 0, stream, false,
                          nullptr);
}

ms_status mamba_trap_scan_workspace_size(const ms_scan_args *args, const void *lambda_raw,
                                         int64_t lambda_batch_stride, int64_t lambda_dim_stride,
                                         const ms_scan_plan *plan, size_t *bytes) {
    if (!bytes) return invalid("bytes is NULL");
    *bytes = 0;
    return trap_scan_impl(args, lambda_raw, lambda_batch_stride, lambda_dim_stride, plan, nullptr, 0, nullptr, true,
                          bytes);
}

ms_status mamba_trap_scan_fwd_ws(const ms_scan_args *args, const void *lambda_raw, int64_t lambda_batch_stride,
                                 int64_t lambda_dim_stride, const ms_scan_plan *plan, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    const CallRange range("mamba_trap_scan_fwd_ws");
    return trap_scan_impl(args, lambda_raw, lambda_batch_stride, lambda_dim_stride, plan, workspace,
                          workspace_bytes, stream, true, nullptr);
}

ms_status mamba_scan_bwd_workspace_size(const ms_scan_args *args, size_t *bytes) {
    if (!bytes) return invalid("bytes is NULL");
    *bytes = 0;
    const ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    *bytes = ms::bwd_workspace_bytes(to_params(args));
    return MS_OK;
}

static ms_status scan_bwd_impl(const ms_scan_args *args, const ms_scan_bwd_args *g, void *workspace,
                               size_t workspace_bytes, void *stream, int ckpt_ready) {
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    if (!g) return invalid("bwd is NULL");
    if (args->seqlen > (int64_t(1) << 30)) return invalid("seqlen above 2^30 is not supported by the backward");
    if (!g->dy || !g->du || !g->ddelta || !g->dA || !g->dB || !g->dC)
        return invalid("dy, du, ddelta, dA, dB and dC are required");
    if ((args->z && !g->dz) || (args->D && !g->dD) || (args->delta_bias && !g->ddelta_bias))
        return invalid("dz, dD and ddelta_bias are required when z, D and delta_bias are given");
    if (g->dy_batch_stride < 0 || g->dy_dim_stride < 0 || g->du_batch_stride < 0 || g->du_dim_stride < 0 ||
        g->ddelta_batch_stride < 0 || g->ddelta_dim_stride < 0 ||
        (g->dz && (g->dz_batch_stride < 0 || g->dz_dim_stride < 0)))
        return invalid("gradient strides must be non-negative");
    const int eb = args->in_dtype == MS_F32 ? 4 : 2;
    if (!elem_aligned(g->dy, eb) || !elem_aligned(g->du, eb) || !elem_aligned(g->ddelta, eb) ||
        (g->dz && !elem_aligned(g->dz, eb)) || !elem_aligned(g->dA, 4) || !elem_aligned(g->dB, 4) ||
        !elem_aligned(g->dC, 4) || (g->dD && !elem_aligned(g->dD, 4)) ||
        (g->ddelta_bias && !elem_aligned(g->ddelta_bias, 4)) ||
        (g->dfinal_state && !elem_aligned(g->dfinal_state, 4)) ||
        (g->dinitial_state && !elem_aligned(g->dinitial_state, 4))) {
        set_error("a gradient pointer is not aligned to its element size");
        return MS_ERR_ALIGNMENT;
    }
    const ms::ScanParams p = to_params(args);
    const size_t need = ms::bwd_workspace_bytes(p);
    if (!workspace || workspace_bytes < need) {
        set_error("%s of %zu bytes needed, %zu given", ckpt_ready ? "checkpoints" : "workspace", need,
                  workspace ? workspace_bytes : static_cast<size_t>(0));
        return MS_ERR_WORKSPACE;
    }
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
        set_error("workspace must be 256-byte aligned");
        return MS_ERR_ALIGNMENT;
    }
    ms::BwdParams q{};
    q.dy = g->dy; q.dy_sb = g->dy_batch_stride; q.dy_sd = g->dy_dim_stride;
    q.dhT = g->dfinal_state;
    q.du = g->du; q.du_sb = g->du_batch_stride; q.du_sd = g->du_dim_stride;
    q.ddelta = g->ddelta; q.dd_sb = g->ddelta_batch_stride; q.dd_sd = g->ddelta_dim_stride;
    q.dz = g->dz; q.dz_sb = g->dz_batch_stride; q.dz_sd = g->dz_dim_stride;
    q.dA = g->dA; q.dB = g->dB; q.dC = g->dC; q.dD = g->dD; q.dbias = g->ddelta_bias;
    q.dh0 = g->dinitial_state;
    q.ckpt = static_cast<float *>(workspace);
    q.ckpt_ready = ckpt_ready;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bc = static_cast<size_t>(args->batch * args->dstate * args->seqlen) * sizeof(float);
    cudaError_t e = cudaMemsetAsync(g->dA, 0, static_cast<size_t>(args->dim * args->dstate) * sizeof(float), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->dB, 0, bc, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->dC, 0, bc, s);
    if (e == cudaSuccess && g->dD) e = cudaMemsetAsync(g->dD, 0, static_cast<size_t>(args->dim) * sizeof(float), s);
    if (e == cudaSuccess && g->ddelta_bias)
        e = cudaMemsetAsync(g->ddelta_bias, 0, static_cast<size_t>(args->dim) * sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the gradient accumulators");
    e = ms::launch_bwd(p, q, args->in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    return MS_OK;
}

ms_status mamba_scan_bwd(const ms_scan_args *args, const ms_scan_bwd_args *g, void *workspace,
                         size_t workspace_bytes, void *stream) {
    const CallRange range("mamba_scan_bwd");
    return scan_bwd_impl(args, g, workspace, workspace_bytes, stream, 0);
}

ms_status mamba_scan_bwd_checkpointed(const ms_scan_args *args, const ms_scan_bwd_args *g,
                                      const float *checkpoints, size_t checkpoint_bytes, void *stream) {
    const CallRange range("mamba_scan_bwd_checkpointed");
    if (!checkpoints) return invalid("checkpoints is NULL");
    return scan_bwd_impl(args, g, const_cast<float *>(checkpoints), checkpoint_bytes, stream, 1);
}

ms_status mamba_scan_fwd_checkpointed(const ms_scan_args *args, float *checkpoints, size_t checkpoint_bytes,
                                      void *workspace, size_t workspace_bytes, void *stream) {
    const CallRange range("mamba_scan_fwd_checkpointed");
    ms_status st = check_scan(args);
    if (st != MS_OK) return st;
    if (!checkpoints) return invalid("checkpoints is NULL");
    const ms::ScanParams p0 = to_params(args);
    const size_t need = ms::bwd_workspace_bytes(p0);
    if (checkpoint_bytes < need) {
        set_error("checkpoints of %zu bytes needed, %zu given", need, checkpoint_bytes);
        return MS_ERR_WORKSPACE;
    }
    if ((reinterpret_cast<uintptr_t>(checkpoints) & 255u) != 0) {
        set_error("checkpoints must be 256-byte aligned");
        return MS_ERR_ALIGNMENT;
    }
    int sms = 0;
    st = device_sms(&sms);
    if (st != MS_OK) return st;
    ms::ScanParams p = p0;
    p.ckpt = checkpoints;   // (the planner then considers the sequential kernels only)
    const ms::ScanPlan plan = ms::plan_scan(p, args->in_dtype, args->force_segments, sms);
    if (plan.kind != 1) {
        set_error("checkpoints are written by the sequential kernels only, which run no forced segments");
        return MS_ERR_UNSUPPORTED;
    }
    return run_plan(p, plan, args->in_dtype, workspace, workspace_bytes, stream);
}

static ms_status check_ssd(const ms_ssd_args *a) {
    if (!a) return invalid("args is NULL");
    if (a->batch <= 0 || a->seqlen <= 0 || a->nheads <= 0 || a->ngroups <= 0)
        return invalid("batch, seqlen, nheads and ngroups must be positive");
    if (a->nheads % a->ngroups != 0) return invalid("nheads must be a multiple of ngroups");
    if (!a->x || !a->dt || !a->B || !a->C || !a->y || !a->A) return invalid("x, dt, B, C, y and A are required");
    if (a->in_dtype != MS_BF16) {
        if (a->in_dtype != MS_F32) return invalid("unknown in_dtype");
        set_error("the SSD kernel takes bf16 inputs only");
        return MS_ERR_UNSUPPORTED;
    }
    if (a->seqlen > (int64_t(1) << 30) || a->batch * a->nheads > (int64_t(1) << 30))
        return invalid("seqlen or batch * nheads too large");
    const int64_t strides[] = {a->x_batch_stride, a->x_token_stride, a->dt_batch_stride, a->dt_token_stride,
                               a->B_batch_stride, a->B_token_stride, a->C_batch_stride, a->C_token_stride,
                               a->y_batch_stride, a->y_token_stride, a->z_batch_stride, a->z_token_stride};
    for (int i = 0; i < (a->z ? 12 : 10); ++i)
        if (strides[i] < 0) return invalid("strides must be non-negative");
    if (a->x_token_stride < a->nheads * MS_SSD_HEADDIM || a->y_token_stride < a->nheads * MS_SSD_HEADDIM ||
        (a->z && a->z_token_stride < a->nheads * MS_SSD_HEADDIM))
        return invalid("the token stride of x, y and z must cover nheads * 64 elements");
    if (a->B_token_stride < a->ngroups * MS_SSD_DSTATE || a->C_token_stride < a->ngroups * MS_SSD_DSTATE)
        return invalid("the token stride of B and C must cover ngroups * 128 elements");
    if (a->dt_token_stride < a->nheads) return invalid("the token stride of dt must cover nheads elements");
    for (int i : {0, 1, 4, 5, 6, 7, 8, 9}) {
        if (strides[i] % 8 != 0) {
            set_error("batch and token strides of x, y, B, C (and z) must be multiples of 8 elements");
            return MS_ERR_ALIGNMENT;
        }
    }
    if (a->z && (a->z_batch_stride % 8 != 0 || a->z_token_stride % 8 != 0)) {
        set_error("batch and token strides of x, y, B, C (and z) must be multiples of 8 elements");
        return MS_ERR_ALIGNMENT;
    }
    if (!elem_aligned(a->x, 16) || !elem_aligned(a->B, 16) || !elem_aligned(a->C, 16) || !elem_aligned(a->y, 16) ||
        (a->z && !elem_aligned(a->z, 16)) || !elem_aligned(a->dt, 2) || !elem_aligned(a->A, 4) ||
        (a->D && !elem_aligned(a->D, 4)) || (a->dt_bias && !elem_aligned(a->dt_bias, 4)) ||
        (a->initial_state && !elem_aligned(a->initial_state, 4)) ||
        (a->final_state && !elem_aligned(a->final_state, 4))) {
        set_error("x, y, B, C and z must be 16-byte aligned, the other pointers aligned to their elements");
        return MS_ERR_ALIGNMENT;
    }
    if (a->withhold_block < 0) return invalid("withhold_block must be >= 0");
    return MS_OK;
}

// CTAs of the persistent schedule the call would take (0: one CTA per (batch, head)).
static ms_status ssd_plan_ctas(const ms_ssd_args *a, int *ctas) {
    int sms = 0;
    const ms_status st = device_sms(&sms);
    if (st != MS_OK) return st;
    *ctas = ms::ssd_persistent_ctas(a->batch, a->nheads, a->seqlen, sms);
    return MS_OK;
}

ms_status mamba_ssd_workspace_size(const ms_ssd_args *a, size_t *bytes) {
    if (!bytes) return invalid("bytes is NULL");
    *bytes = 0;
    ms_status st = check_ssd(a);
    if (st != MS_OK) return st;
    int ctas = 0;
    st = ssd_plan_ctas(a, &ctas);
    if (st != MS_OK) return st;
    *bytes = ctas ? ms::ssd_persistent_ws_bytes(ctas) : static_cast<size_t>(MS_SSD_WORKSPACE_BYTES);
    return MS_OK;
}

ms_status mamba_ssd_fwd(const ms_ssd_args *a, void *workspace, size_t workspace_bytes, void *stream) {
    const CallRange range("mamba_ssd_fwd");
    ms_status st = check_ssd(a);
    if (st != MS_OK) return st;
    if (!workspace || workspace_bytes < MS_SSD_WORKSPACE_BYTES) {
        set_error("workspace of %d bytes needed, %zu given", MS_SSD_WORKSPACE_BYTES,
                  workspace ? workspace_bytes : static_cast<size_t>(0));
        return MS_ERR_WORKSPACE;
    }
    if (!elem_aligned(workspace, 16)) {
        set_error("workspace must be 16-byte aligned");
        return MS_ERR_ALIGNMENT;
    }
    ms::SsdParams p{};
    p.x = a->x; p.x_sb = a->x_batch_stride; p.x_st = a->x_token_stride;
    p.dt = a->dt; p.dt_sb = a->dt_batch_stride; p.dt_st = a->dt_token_stride;
    p.B = a->B; p.B_sb = a->B_batch_stride; p.B_st = a->B_token_stride;
    p.C = a->C; p.C_sb = a->C_batch_stride; p.C_st = a->C_token_stride;
    p.z = a->z; p.z_sb = a->z_batch_stride; p.z_st = a->z_token_stride;
    p.y = a->y; p.y_sb = a->y_batch_stride; p.y_st = a->y_token_stride;
    p.A = a->A; p.D = a->D; p.dt_bias = a->dt_bias; p.h0 = a->initial_state; p.hT = a->final_state;
    p.batch = a->batch; p.seqlen = a->seqlen; p.nheads = a->nheads; p.ngroups = a->ngroups;
    p.softplus = a->dt_softplus ? 1 : 0;
    p.status = static_cast<int *>(workspace);
    p.wait_limit_ns = a->wait_limit_us ? 1000ull * a->wait_limit_us : 1000000000ull;
    p.withhold_block = a->withhold_block;
    int ctas = 0;
    st = ssd_plan_ctas(a, &ctas);
    if (st != MS_OK) return st;
    if (ctas > 0 && workspace_bytes >= ms::ssd_persistent_ws_bytes(ctas)) {
        p.sk_ctas = ctas;
        p.sk_flag = reinterpret_cast<int *>(static_cast<char *>(workspace) + ms::ssd_flag_offset());
        p.sk_carry = reinterpret_cast<float *>(static_cast<char *>(workspace) + ms::ssd_carry_offset(ctas));
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = ms::launch_ssd(p, s);
    if (e == cudaErrorNotSupported) {
        set_error("the driver offers no tensor-map encoder");
        return MS_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return cuda_fail(e, "SSD kernel launch");
    return MS_OK;
}

}  // extern "C"
