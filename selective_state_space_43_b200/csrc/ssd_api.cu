// ssd_api.cu -- the extern "C" entry points declared in include/ssd.h:
// argument validation (before any launch), kernel-path choice, launches.
#include <stdint.h>

#include "ssd.h"
#include "ssd_backward.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_mimo.h"

namespace {

thread_local ssd::TimingHook g_hook;
thread_local uint64_t g_test_stall_ns = 0;  // ssd_test_stall_prefill

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ssd_status check_dims(const ssd_dims* d, ssd_dtype dtype, bool prefill) {
    if (!d) return SSD_ERR_NULL;
    if (dtype != SSD_F32 && dtype != SSD_BF16 && dtype != SSD_BF16_YF32) return SSD_ERR_DTYPE;
    if (d->batch < 0 || (prefill && d->seqlen < 0)) return SSD_ERR_SHAPE;
    if (d->nheads <= 0 || d->ngroups <= 0 || d->nheads % d->ngroups != 0) return SSD_ERR_SHAPE;
    if (d->headdim != 64) return SSD_ERR_SHAPE;
    if (!(d->d_state == 16 || d->d_state == 32 || d->d_state == 64 || d->d_state == 128)) return SSD_ERR_SHAPE;
    if (d->d_conv != 4) return SSD_ERR_SHAPE;
    if (prefill && !(d->chunk == 64 || d->chunk == 128)) return SSD_ERR_SHAPE;
    // index arithmetic inside the kernels uses 32-bit per-token offsets
    const int64_t conv_dim = (int64_t)d->nheads * d->headdim + 2LL * d->ngroups * d->d_state;
    if (conv_dim > (1LL << 24)) return SSD_ERR_SHAPE;
    if (d->batch * (int64_t)d->nheads > (1LL << 31) - 1) return SSD_ERR_SHAPE;
    return SSD_OK;
}

// Each input row stride must cover its row and keep rows 16-byte aligned (tensor maps, vector loads).
ssd_status check_strides(const ssd_row_strides& r, const ssd::Shape& s, ssd_dtype dtype) {
    const int64_t esz = dtype == SSD_F32 ? 4 : 2;
    const int64_t st[5] = {r.x, r.z, r.dt, r.B, r.C}, w[5] = {s.HP, s.HP, s.H, s.GN, s.GN};
    for (int k = 0; k < 5; ++k) {
        if (st[k] < w[k]) return SSD_ERR_SHAPE;
        if ((st[k] * esz) % 16 != 0) return SSD_ERR_ALIGN;
    }
    return SSD_OK;
}

ssd_status check_params(const ssd_params* p) {
    if (!p || !p->A || !p->D || !p->dt_bias || !p->conv_w || !p->conv_b) return SSD_ERR_NULL;
    if (!aligned16(p->A) || !aligned16(p->D) || !aligned16(p->dt_bias) || !aligned16(p->conv_w) ||
        !aligned16(p->conv_b))
        return SSD_ERR_ALIGN;
    return SSD_OK;
}

// A byte range [p, p + n) of a caller's buffer (p may be null: no buffer).
struct Span {
    const void* p;
    uint64_t n;
};

bool overlap(const Span& a, const Span& b) {
    if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.n && b0 < a0 + a.n;
}

// Whether any output range overlaps another output or any input range.
bool outputs_alias(const Span* outs, int nout, const Span* ins, int nin) {
    for (int i = 0; i < nout; ++i) {
        for (int j = i + 1; j < nout; ++j)
            if (overlap(outs[i], outs[j])) return true;
        for (int j = 0; j < nin; ++j)
            if (overlap(outs[i], ins[j])) return true;
    }
    return false;
}

}  // namespace

extern "C" {

const char* ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "ok";
        case SSD_ERR_NULL: return "a required pointer is NULL";
        case SSD_ERR_SHAPE: return "unsupported or inconsistent sizes";
        case SSD_ERR_DTYPE: return "unknown activation dtype";
        case SSD_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case SSD_ERR_UNSUPPORTED: return "valid but unsupported arguments (aliasing outputs)";
        case SSD_ERR_CUDA: return "a CUDA runtime call failed";
        case SSD_ERR_WORKSPACE: return "workspace missing or too small";
        case SSD_ERR_TIMEOUT: return "a bounded device-side wait gave up";
        case SSD_ERR_RANGE: return "a backward operand beyond fp16 range (the gradients of that call are invalid)";
    }
    return "unknown status";
}

const char* ssd_version(void) { return "ssd_b200 1.0 (sm_100a)"; }

int ssd_prefill_path(const ssd_dims* d, ssd_dtype dtype) {
    const ssd_status st = check_dims(d, dtype, true);
    if (st != SSD_OK) return -(int)st;
    return ssd::prefill_tc_supported(d->headdim, d->d_state, d->chunk, d->nheads, dtype != SSD_F32) ? 1 : 2;
}

size_t ssd_prefill_workspace_bytes(const ssd_dims* d, ssd_dtype dtype) {
    if (ssd_prefill_path(d, dtype) != 1) return 0;
    return ssd::prefill_tc_workspace_bytes(d->batch, d->seqlen, d->ngroups, d->d_state);
}

// ssd_prefill with optional input row strides (nullptr: contiguous rows).
static ssd_status prefill_impl(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params,
                               const ssd_row_strides* rs, const void* x, const void* dt, const void* B,
                               const void* C, const void* z, const float* init_state, const void* init_conv_state,
                               void* y, float* final_state, void* conv_state, void* workspace,
                               size_t workspace_bytes, void* stream) {
    ssd_status st = check_dims(d, dtype, true);
    if (st != SSD_OK) return st;
    if ((st = check_params(params)) != SSD_OK) return st;
    // with no tokens the activations and y are never touched and may be NULL
    const bool tokens = d->batch > 0 && d->seqlen > 0;
    if (tokens && (!x || !dt || !B || !C || !z || !y)) return SSD_ERR_NULL;
    if (d->batch > 0 && (!final_state || !conv_state)) return SSD_ERR_NULL;
    const void* ptrs[] = {x, dt, B, C, z, init_state, init_conv_state, y, final_state, conv_state, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    if ((tokens && (y == x || y == z)) || (init_conv_state && init_conv_state == conv_state))
        return SSD_ERR_UNSUPPORTED;
    const ssd::Shape s = ssd::make_shape(*d);
    ssd_row_strides r{s.HP, s.HP, s.H, s.GN, s.GN};
    if (rs) {
        if ((st = check_strides(*rs, s, dtype)) != SSD_OK) return st;
        r = *rs;
    }
    const int path = ssd_prefill_path(d, dtype);
    const size_t need = path == 1 ? ssd::prefill_tc_workspace_bytes(d->batch, d->seqlen, d->ngroups, d->d_state) : 0;
    if (need > 0 && (!workspace || workspace_bytes < need)) return SSD_ERR_WORKSPACE;
    if (d->batch == 0) return SSD_OK;

    ssd::PrefillArgs a;
    a.batch = s.batch;
    a.L = s.seqlen;
    a.nchunks = s.nchunks;
    a.H = s.H; a.P = s.P; a.N = s.N; a.G = s.G; a.Q = s.Q;
    a.HP = s.HP; a.GN = s.GN; a.conv_dim = s.conv_dim; a.hpg = s.heads_per_group;
    a.A = params->A; a.D = params->D; a.dt_bias = params->dt_bias;
    a.conv_w = params->conv_w; a.conv_b = params->conv_b;
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z;
    a.init_state = init_state; a.init_conv_state = init_conv_state;
    a.y = y; a.final_state = final_state; a.conv_state = conv_state;
    a.workspace = workspace;
    a.rs_x = r.x; a.rs_z = r.z; a.rs_dt = r.dt; a.rs_B = r.B; a.rs_C = r.C;
    a.stall_ns = g_test_stall_ns;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const ssd::ActKind kind = dtype == SSD_F32 ? ssd::ActKind::F32 : (dtype == SSD_BF16 ? ssd::ActKind::BF16
                                                                                        : ssd::ActKind::BF16_YF32);
    cudaError_t e = path == 1 ? ssd::launch_prefill_tc(a, kind, cs, g_hook)
                              : ssd::launch_prefill_simt(a, kind, cs, g_hook);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_prefill(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params, const void* x,
                       const void* dt, const void* B, const void* C, const void* z, const float* init_state,
                       const void* init_conv_state, void* y, float* final_state, void* conv_state,
                       void* workspace, size_t workspace_bytes, void* stream) {
    return prefill_impl(d, dtype, params, nullptr, x, dt, B, C, z, init_state, init_conv_state, y, final_state,
                        conv_state, workspace, workspace_bytes, stream);
}

ssd_status ssd_prefill_strided(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params,
                               const ssd_row_strides* row_strides, const void* x, const void* dt, const void* B,
                               const void* C, const void* z, const float* init_state, const void* init_conv_state,
                               void* y, float* final_state, void* conv_state, void* workspace,
                               size_t workspace_bytes, void* stream) {
    return prefill_impl(d, dtype, params, row_strides, x, dt, B, C, z, init_state, init_conv_state, y,
                        final_state, conv_state, workspace, workspace_bytes, stream);
}

size_t ssd_prefill_varlen_workspace_bytes(const ssd_dims* d, ssd_dtype dtype) {
    if (ssd_prefill_path(d, dtype) != 1) return 0;
    return ssd::prefill_tc_workspace_bytes(1, d->seqlen, d->ngroups, d->d_state);  // post-conv B/C of all rows
}

ssd_status ssd_prefill_varlen(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params,
                              const int64_t* cu_seqlens, const void* x, const void* dt, const void* B,
                              const void* C, const void* z, const float* init_state, const void* init_conv_state,
                              void* y, float* final_state, void* conv_state, void* workspace,
                              size_t workspace_bytes, void* stream) {
    ssd_status st = check_dims(d, dtype, true);
    if (st != SSD_OK) return st;
    if ((st = check_params(params)) != SSD_OK) return st;
    if (d->seqlen > (1LL << 31) - 256) return SSD_ERR_SHAPE;  // tensor-map row coordinates are 32-bit
    if (!cu_seqlens && d->batch > 0) return SSD_ERR_NULL;
    const bool tokens = d->seqlen > 0;
    if (tokens && (!x || !dt || !B || !C || !z || !y)) return SSD_ERR_NULL;
    if (d->batch > 0 && (!final_state || !conv_state)) return SSD_ERR_NULL;
    const void* ptrs[] = {x, dt, B, C, z, init_state, init_conv_state, y, final_state, conv_state, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(cu_seqlens) & 7u) return SSD_ERR_ALIGN;
    if ((tokens && (y == x || y == z)) || (init_conv_state && init_conv_state == conv_state))
        return SSD_ERR_UNSUPPORTED;
    const int path = ssd_prefill_path(d, dtype);
    const size_t need = ssd_prefill_varlen_workspace_bytes(d, dtype);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SSD_ERR_WORKSPACE;
    if (d->batch == 0) return SSD_OK;
    int* err = ssd::device_error_flag();
    if (!err) return SSD_ERR_CUDA;

    const ssd::Shape s = ssd::make_shape(*d);
    ssd::PrefillArgs a;
    a.batch = s.batch;
    a.L = s.seqlen;  // all rows
    a.nchunks = s.nchunks;
    a.H = s.H; a.P = s.P; a.N = s.N; a.G = s.G; a.Q = s.Q;
    a.HP = s.HP; a.GN = s.GN; a.conv_dim = s.conv_dim; a.hpg = s.heads_per_group;
    a.A = params->A; a.D = params->D; a.dt_bias = params->dt_bias;
    a.conv_w = params->conv_w; a.conv_b = params->conv_b;
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z;
    a.init_state = init_state; a.init_conv_state = init_conv_state;
    a.y = y; a.final_state = final_state; a.conv_state = conv_state;
    a.workspace = workspace;
    a.cu = cu_seqlens;
    a.err = err;
    a.rs_x = s.HP; a.rs_z = s.HP; a.rs_dt = s.H; a.rs_B = s.GN; a.rs_C = s.GN;
    a.stall_ns = g_test_stall_ns;
    const ssd::ActKind kind = dtype == SSD_F32 ? ssd::ActKind::F32 : (dtype == SSD_BF16 ? ssd::ActKind::BF16
                                                                                        : ssd::ActKind::BF16_YF32);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = path == 1 ? ssd::launch_prefill_tc(a, kind, cs, g_hook)
                              : ssd::launch_prefill_simt(a, kind, cs, g_hook);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_decode_step(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params, const void* x,
                           const void* dt, const void* B, const void* C, const void* z, void* conv_state,
                           float* ssm_state, void* y, void* stream) {
    ssd_status st = check_dims(d, dtype, false);
    if (st != SSD_OK) return st;
    if ((st = check_params(params)) != SSD_OK) return st;
    if (!x || !dt || !B || !C || !z || !conv_state || !ssm_state || !y) return SSD_ERR_NULL;
    const void* ptrs[] = {x, dt, B, C, z, conv_state, ssm_state, y};
    for (const void* p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    if (y == x || y == z) return SSD_ERR_UNSUPPORTED;
    if (d->batch == 0) return SSD_OK;
    const ssd::Shape s = ssd::make_shape(*d);
    ssd::DecodeArgs a;
    a.H = s.H; a.P = s.P; a.N = s.N; a.G = s.G; a.HP = s.HP; a.GN = s.GN;
    a.conv_dim = s.conv_dim; a.hpg = s.heads_per_group;
    a.A = params->A; a.D = params->D; a.dt_bias = params->dt_bias;
    a.conv_w = params->conv_w; a.conv_b = params->conv_b;
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z;
    a.conv_state = conv_state; a.ssm_state = ssm_state; a.y = y;
    const ssd::ActKind kind = dtype == SSD_F32 ? ssd::ActKind::F32 : (dtype == SSD_BF16 ? ssd::ActKind::BF16
                                                                                        : ssd::ActKind::BF16_YF32);
    cudaError_t e = ssd::launch_decode(a, s.batch, kind, static_cast<cudaStream_t>(stream), g_hook);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

size_t ssd_prefill_backward_workspace_bytes(const ssd_dims* d) {
    if (!d || check_dims(d, SSD_F32, true) != SSD_OK) return 0;
    return ssd::bwd::workspace_bytes(d->batch, d->seqlen, d->nheads, d->headdim, d->d_state, d->ngroups);
}

ssd_status ssd_prefill_backward(const ssd_dims* d, ssd_dtype dtype, const ssd_params* params, const void* x,
                                const void* dt, const void* B, const void* C, const void* z,
                                const float* init_state, const void* init_conv_state, const void* dy,
                                const float* d_final_state, const ssd_grads* g, void* workspace,
                                size_t workspace_bytes, void* stream) {
    ssd_status st = check_dims(d, dtype, true);
    if (st != SSD_OK) return st;
    if ((st = check_params(params)) != SSD_OK) return st;
    if (!g) return SSD_ERR_NULL;
    // grid limits of the backward's launches: 64-token chunks and the batch on the y / z grid axes
    if ((d->seqlen + 63) / 64 > 65535 || d->batch > 65535) return SSD_ERR_SHAPE;
    const bool tokens = d->batch > 0 && d->seqlen > 0;
    if (tokens && (!x || !dt || !B || !C || !z || !dy || !g->dx || !g->ddt || !g->dB || !g->dC || !g->dz))
        return SSD_ERR_NULL;
    if (!g->dA || !g->dD || !g->ddt_bias || !g->dconv_w || !g->dconv_b) return SSD_ERR_NULL;
    const void* ptrs[] = {x, dt, B, C, z, init_state, init_conv_state, dy, d_final_state, g->dx, g->ddt, g->dB,
                          g->dC, g->dz, g->dA, g->dD, g->ddt_bias, g->dconv_w, g->dconv_b, g->d_init_state,
                          g->d_init_conv_state, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    const size_t need = ssd::bwd::workspace_bytes(d->batch, d->seqlen, d->nheads, d->headdim, d->d_state,
                                                  d->ngroups);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SSD_ERR_WORKSPACE;
    {
        const uint64_t rows = (uint64_t)d->batch * (uint64_t)d->seqlen, H = d->nheads;
        const uint64_t HP = H * d->headdim, GN = (uint64_t)d->ngroups * d->d_state, cd = HP + 2 * GN;
        const uint64_t st = (uint64_t)d->batch * HP * d->d_state, ae = dtype == SSD_F32 ? 4 : 2;
        const uint64_t de = dtype == SSD_BF16 ? 2 : 4;
        const Span ins[] = {{x, rows * HP * ae},         {dt, rows * H * ae},          {B, rows * GN * ae},
                            {C, rows * GN * ae},         {z, rows * HP * ae},          {dy, rows * HP * de},
                            {init_state, st * 4},        {init_conv_state, (uint64_t)d->batch * cd * 3 * ae},
                            {d_final_state, st * 4},     {params->A, H * 4},           {params->D, H * 4},
                            {params->dt_bias, H * 4},    {params->conv_w, cd * 16},    {params->conv_b, cd * 4},
                            {workspace, need}};
        const Span outs[] = {{g->dx, rows * HP * 4},     {g->ddt, rows * H * 4},       {g->dB, rows * GN * 4},
                             {g->dC, rows * GN * 4},     {g->dz, rows * HP * 4},       {g->dA, H * 4},
                             {g->dD, H * 4},             {g->ddt_bias, H * 4},         {g->dconv_w, cd * 16},
                             {g->dconv_b, cd * 4},       {g->d_init_state, st * 4},
                             {g->d_init_conv_state, (uint64_t)d->batch * cd * 3 * 4}};
        if (outputs_alias(outs, 12, ins, 15)) return SSD_ERR_UNSUPPORTED;
    }

    ssd::bwd::BwdArgs a{};
    a.batch = d->batch;
    a.L = d->seqlen;
    a.H = d->nheads; a.P = d->headdim; a.N = d->d_state; a.G = d->ngroups;
    a.act_bf16 = dtype != SSD_F32;
    a.dy_bf16 = dtype == SSD_BF16;
    a.A = params->A; a.D = params->D; a.dt_bias = params->dt_bias;
    a.conv_w = params->conv_w; a.conv_b = params->conv_b;
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z; a.dy = dy;
    a.init_state = init_state; a.init_conv_state = init_conv_state; a.d_final = d_final_state;
    a.dx = g->dx; a.ddt = g->ddt; a.dB = g->dB; a.dC = g->dC; a.dz = g->dz;
    a.dA = g->dA; a.dD = g->dD; a.ddt_bias = g->ddt_bias; a.dconv_w = g->dconv_w; a.dconv_b = g->dconv_b;
    a.d_init_state = g->d_init_state; a.d_init_conv_state = g->d_init_conv_state;
    a.workspace = workspace;
    a.ev_before = g_hook.ev_before;
    a.ev_after = g_hook.ev_after;
    cudaError_t e = ssd::bwd::launch_prefill_backward(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_mimo_decode_step(const ssd_dims* d, int32_t rank, ssd_dtype dtype, const ssd_params* params,
                                const void* x, const void* dt, const void* B, const void* C, const void* z,
                                float* ssm_state, void* y, void* stream) {
    ssd_status st = check_dims(d, dtype, false);
    if (st != SSD_OK) return st;
    if (!(rank == 1 || rank == 2 || rank == 4 || rank == 8)) return SSD_ERR_SHAPE;
    if (!params || !params->A || !params->D || !params->dt_bias) return SSD_ERR_NULL;
    if (!aligned16(params->A) || !aligned16(params->D) || !aligned16(params->dt_bias)) return SSD_ERR_ALIGN;
    if (!x || !dt || !B || !C || !z || !ssm_state || !y) return SSD_ERR_NULL;
    const void* ptrs[] = {x, dt, B, C, z, ssm_state, y};
    for (const void* p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    {
        const uint64_t bh = (uint64_t)d->batch * d->nheads, ae = dtype == SSD_F32 ? 4 : 2;
        const uint64_t ye = dtype == SSD_BF16 ? 2 : 4, R = (uint64_t)rank;
        const uint64_t bc = (uint64_t)d->batch * d->ngroups * R * d->d_state * ae;
        const Span ins[] = {{x, bh * R * d->headdim * ae}, {dt, bh * ae}, {B, bc}, {C, bc},
                            {z, bh * R * d->headdim * ae}, {ssm_state, bh * d->headdim * d->d_state * 4}};
        const Span outs[] = {{y, bh * R * d->headdim * ye}};
        if (outputs_alias(outs, 1, ins, 6)) return SSD_ERR_UNSUPPORTED;
    }
    if (d->batch == 0) return SSD_OK;
    ssd::mimo::MimoArgs a{};
    a.batch = d->batch;
    a.H = d->nheads; a.P = d->headdim; a.N = d->d_state; a.G = d->ngroups; a.R = rank;
    a.act_bf16 = dtype != SSD_F32;
    a.y_bf16 = dtype == SSD_BF16;
    a.A = params->A; a.D = params->D; a.dt_bias = params->dt_bias;
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.z = z;
    a.ssm_state = ssm_state;
    a.y = y;
    a.ev_before = g_hook.ev_before;
    a.ev_after = g_hook.ev_after;
    cudaError_t e = ssd::mimo::launch_mimo_decode(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_device_status(void* stream) {
    int flag = 0;
    if (ssd::read_and_clear_tc_error(&flag, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SSD_ERR_CUDA;
    int mimo_flag = 0, bwd_flag = 0, chunk_bwd_flag = 0, decode_flag = 0;
    if (ssd::read_and_clear_decode_error(&decode_flag) != cudaSuccess) return SSD_ERR_CUDA;
    if (ssd::mimo::read_and_clear_mimo_error(&mimo_flag) != cudaSuccess) return SSD_ERR_CUDA;
    if (ssd::bwd::read_and_clear_bwd_tc_error(&bwd_flag) != cudaSuccess) return SSD_ERR_CUDA;
    if (ssd::bwd::read_and_clear_chunk_bwd_tc_error(&chunk_bwd_flag) != cudaSuccess) return SSD_ERR_CUDA;
    // the backward kernels' words: bit 0 a bounded wait gave up, bit 1 an operand beyond fp16 range
    if ((flag & ssd::kErrTimeout) || mimo_flag || decode_flag || ((bwd_flag | chunk_bwd_flag) & 1)) return SSD_ERR_TIMEOUT;
    if ((bwd_flag | chunk_bwd_flag) & 2) return SSD_ERR_RANGE;
    return flag & ssd::kErrBadSeqlens ? SSD_ERR_SHAPE : SSD_OK;
}

ssd_status ssd_test_stall_prefill(uint64_t wait_ns) {
    g_test_stall_ns = wait_ns;
    return SSD_OK;
}

ssd_status ssd_set_timing_events(void* before_main, void* after_main) {
    if ((before_main == nullptr) != (after_main == nullptr)) return SSD_ERR_NULL;
    g_hook.ev_before = static_cast<cudaEvent_t>(before_main);
    g_hook.ev_after = static_cast<cudaEvent_t>(after_main);
    return SSD_OK;
}

}  // extern "C"
