// Internal host-side interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ms {

// Everything a scan kernel reads, in one by-value kernel parameter.
struct ScanParams {
    int64_t batch, dim, dstate, seqlen;
    const void *u;     int64_t u_sb, u_sd;
    const void *delta; int64_t dl_sb, dl_sd;
    const void *B;     int64_t B_sb, B_sn;
    const void *C;     int64_t C_sb, C_sn;
    const void *z;     int64_t z_sb, z_sd;
    void *y;           int64_t y_sb, y_sd;
    const float *A, *D, *delta_bias, *h0;
    float *hT;
    int softplus;
    int nseg;           // segments per row (1 = no multi-block carry)
    int64_t seg_len;    // time steps per segment, a multiple of the chunk length
    float *ws_P;        // (batch*dim, nseg, 16): decay product of each segment
    float *ws_H;        // (batch*dim, nseg, 16): end state of each segment from zero
    // Convolution prologue (sequential kernels only): when conv_w is set, u
    // holds the convolution input x and the SSM input is
    // act(conv_b[d] + sum_k conv_w[d*conv_width + k] x[t - conv_width + 1 + k]).
    const float *conv_w, *conv_b;
    int conv_width, conv_silu;
    // Exponential-trapezoidal recurrence (sequential kernels only): when set,
    // lambda = sigmoid(lambda_raw) per (b, d, t) mixes the previous and the
    // current input, h_t = a_t h_{t-1} + (1-lambda_t) delta_t a_t B_{t-1} u_{t-1}
    // + lambda_t delta_t B_t u_t.
    const void *lambda_raw; int64_t lm_sb, lm_sd;
    // Checkpoints for the backward pass (sequential kernels, plain scan only):
    // when set, the state after every 8th step, (batch*dim, ceil(L/8), 16)
    // float32, as the backward's workspace lays it out.
    float *ckpt;
    // Persistent schedule of the sequential kernels (sk_ctas > 0): the chunks
    // of all units (one batch entry x one block of rows) form one list, cut
    // into sk_ctas equal ranges, one per CTA. A unit whose chunks fall into two
    // ranges is started by the CTA that owns its first chunks and continued by
    // the next CTA from the state left in sk_carry (ready when sk_flag[unit] is
    // set). sk_ctas == 0: one CTA per unit.
    int sk_ctas;
    int sk_units;             // batch * row blocks
    float *sk_carry;          // (units, rows per unit, 16) states handed over
    int *sk_flag;             // (units) zero at launch, 1 once the unit's carry is written
    int *sk_status;           // receives MS_ERR_TIMEOUT if a carry wait gave up
};

// Launch configuration chosen on the host for one scan call.
struct ScanPlan {
    int kind;           // 0: chunked kernels (scan_fwd.cu); 1: sequential kernels (scan_rec.cu)
    int lg;             // kind 0: lanes that share one row pair's chunk (4, 8 or 16);
                        // kind 1: lanes per row (2, 4, 8 or 16)
    int config;         // index of the compiled kernel configuration
    int warps;          // warps per CTA
    int rows_per_cta;   // warps * (32 / lg)
    int chunk;          // time steps per chunk = lg * 8
    int vec;            // 1 if every row start is 16-byte aligned (vector path)
    int nseg;
    int64_t seg_len;
    size_t ws_bytes;
    int ctas;           // kind 1: 0 = one CTA per unit; > 0 = persistent schedule over this many CTAs
    int iow;            // kind 1: I/O warps per CTA (2 or 4)
};

// Workspace of a persistent sequential scan: a status word (first 256 bytes),
// the units' carry flags, then their carry states; everything before the
// carry states is cleared on the stream before each launch.
size_t rec_persistent_ws_bytes(int64_t units, int rows_per_unit);
size_t rec_persistent_clear_bytes(int64_t units);
// Point p's persistent-schedule fields into the workspace `ws`.
void rec_bind_workspace(ScanParams &p, void *ws, int64_t units, int ctas);

// With p.conv_w or p.lambda_raw set only the sequential configurations that
// fuse the convolution prologue or run the trapezoidal rule (lanes 2 and 4)
// are considered.
// persistent_ok: the caller can provide the persistent schedule's workspace.
ScanPlan plan_scan(const ScanParams &p, int in_dtype, int force_segments, int num_sms, bool persistent_ok = true);
// A plan with a fixed configuration, CTA size and segment count; returns false
// (and leaves `out` unspecified) when the configuration cannot run `p`.
// ctas: sequential configurations only, 0 = one CTA per unit, > 0 = persistent
// schedule over that many CTAs (at most rec_max_ctas).
bool make_plan(const ScanParams &p, int in_dtype, int config, int warps, int segments, int ctas, int num_sms,
               ScanPlan *out);
// Point the kernel parameters at the plan's workspace (multi-block carry, or
// the persistent schedule's flags and carry states).
void bind_workspace(ScanParams &p, const ScanPlan &plan, void *workspace);
int scan_num_configs();
bool scan_config_info(int config, int *lanes, int *states_per_pass, int *max_warps);
int scan_config_kind(int config);   // 0 chunked, 1 sequential, -1 unknown index
cudaError_t launch_scan(const ScanParams &p, const ScanPlan &plan, int in_dtype,
                        cudaStream_t stream);

// Sequential kernels (scan_rec.cu): CTAs of rec_threads() threads (recurrence
// and I/O warps) owning rec_rows(lanes_per_row) rows, no workspace, one segment.
// Variants of the sequential kernel: 0 plain, 1 convolution prologue, 2 trapezoidal rule.
// iow: I/O warps per CTA (2, or 4 for the plain scan with 2, 4 or 8 lanes per row).
int rec_variant(const ScanParams &p);
int rec_smem_bytes(int in_dtype, int lanes_per_row, int variant, int iow);
int rec_chunk();
int rec_threads(int iow);
int rec_rows(int lanes_per_row);
int rec_ctas_per_sm(int in_dtype, int lanes_per_row, bool vec, int variant, int iow);
bool rec_supports_variant(int lanes_per_row, int variant, int iow);
cudaError_t launch_rec(const ScanParams &p, int lanes_per_row, bool vec, int in_dtype, int iow,
                       cudaStream_t stream);
// Largest CTA count a persistent sequential launch can use (every CTA resident
// at once, at most one per unit).
int rec_max_ctas(const ScanParams &p, int in_dtype, int lanes_per_row, bool vec, int num_sms, int iow);

// Backward pass (scan_bwd.cu): output gradients in, input gradients out.
// du, ddelta, dz: (batch, dim, L) in the input dtype; dB, dC: (batch, dstate,
// L) float32 contiguous; dA (dim, dstate), dD and dbias (dim), dh0 (batch,
// dim, dstate) float32. dA, dB, dC, dD and dbias are accumulated with atomics
// and must be zero before the launch. ckpt: bwd_workspace_bytes(p) bytes.
struct BwdParams {
    const void *dy;    int64_t dy_sb, dy_sd;
    const float *dhT;
    void *du;          int64_t du_sb, du_sd;
    void *ddelta;      int64_t dd_sb, dd_sd;
    void *dz;          int64_t dz_sb, dz_sd;
    float *dA, *dB, *dC, *dD, *dbias, *dh0;
    float *ckpt;
    int ckpt_ready;   // ckpt already holds the checkpoints (written by the forward): skip the forward sweep
};
size_t bwd_workspace_bytes(const ScanParams &p);
cudaError_t launch_bwd(const ScanParams &p, const BwdParams &q, int in_dtype, cudaStream_t stream);

struct UpdateParams {
    int64_t batch, dim, dstate;
    float *state;      int64_t s_sb, s_sd;
    const void *x;     int64_t x_sb;
    const void *delta; int64_t dl_sb;
    const void *B;     int64_t B_sb;
    const void *C;     int64_t C_sb;
    const void *z;     int64_t z_sb;
    void *y;           int64_t y_sb;
    const float *A, *D, *delta_bias;
    int softplus;
    // Convolution prologue: when conv_w is set, x is the convolution input and
    // conv_state (batch, dim, conv_width; element strides cs_sb, cs_sd, the
    // width axis contiguous) holds the last conv_width inputs, oldest first.
    void *conv_state;  int64_t cs_sb, cs_sd;
    const float *conv_w, *conv_b;
    int conv_width, conv_silu;
};

cudaError_t launch_state_update(const UpdateParams &p, int in_dtype, cudaStream_t stream);

// Mamba-2 scalar-decay SSM (SSD) forward, bf16 inputs, headdim 64, dstate 128.
// x and z, y: (batch, seqlen, nheads, 64), the last two axes contiguous, batch
// and token element strides *_sb, *_st. dt: (batch, seqlen, nheads), head
// axis contiguous. B, C: (batch, seqlen, ngroups, 128), the last two axes
// contiguous. h0 / hT: (batch, nheads, 64, 128) float32 contiguous or null.
// status: a device int that receives MS_ERR_TIMEOUT if a pipeline wait of
// the kernel gave up (it is not cleared by the launch).
struct SsdParams {
    const void *x;     int64_t x_sb, x_st;
    const void *dt;    int64_t dt_sb, dt_st;
    const void *B;     int64_t B_sb, B_st;
    const void *C;     int64_t C_sb, C_st;
    const void *z;     int64_t z_sb, z_st;
    void *y;           int64_t y_sb, y_st;
    const float *A, *D, *dt_bias, *h0;
    float *hT;
    int64_t batch, seqlen, nheads, ngroups;
    int softplus;
    int *status;
    uint64_t wait_limit_ns;   // limit of each pipeline wait
    int withhold_block;       // tests: k > 0 withholds block k - 1's loads (the wait for them runs out)
    // Persistent schedule (sk_ctas > 0): the chunks of all (batch, head) pairs
    // form one list cut evenly over sk_ctas resident CTAs; CTA g hands the
    // state at the end of its first piece to CTA g + 1 through sk_carry[g]
    // (64 x 128 floats) and raises sk_flag[g]. 0: one CTA per (batch, head).
    int sk_ctas;
    int *sk_flag;
    float *sk_carry;
};
constexpr int kSsdHeadDim = 64;
constexpr int kSsdState = 128;
constexpr int kSsdChunk = 128;
// Encodes the kernel's tensor maps and launches it (cooperatively for the
// persistent schedule, after clearing the status word and the carry flags).
// Returns cudaErrorNotSupported when the driver offers no tensor-map encoder.
cudaError_t launch_ssd(const SsdParams &p, cudaStream_t stream);
// CTAs of the persistent schedule for these sizes on num_sms SMs (one CTA per
// SM), or 0 when one CTA per (batch, head) does as well.
int ssd_persistent_ctas(int64_t batch, int64_t nheads, int64_t seqlen, int num_sms);
// Workspace bytes of the persistent schedule over ctas CTAs (status word,
// flags and carries).
size_t ssd_persistent_ws_bytes(int ctas);
// Offsets of the flags and the carries in that workspace.
size_t ssd_flag_offset();
size_t ssd_carry_offset(int ctas);

// Record the message that mamba_last_error() returns on this thread.
void record_error(const char *fmt, ...);

}  // namespace ms
