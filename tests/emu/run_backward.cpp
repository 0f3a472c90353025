// run_backward.cpp -- runs the backward kernels of ssd_backward.cu on the CPU through the host
// emulation in emu_cuda.h (built with AddressSanitizer by the tests; never part of the library).
//
// usage: run_backward <in.bin> <out.bin>
// in.bin:  11 int64 (batch, L, H, P, N, G, act_bf16, dy_bf16, has_init_state, has_init_conv_state,
//          has_d_final), then the arrays in this order, each in its own dtype:
//          A, D, dt_bias [H] f32; conv_w [conv_dim][4] f32; conv_b [conv_dim] f32;
//          x [B][L][H*P], dt [B][L][H], B [B][L][G*N], C [B][L][G*N], z [B][L][H*P] (act dtype);
//          dy [B][L][H*P] (dy dtype); init_state [B][H][P][N] f32; init_conv_state [B][conv_dim][3]
//          (act dtype); d_final [B][H][P][N] f32 (the last three only if present).
// out.bin: f32 dx, ddt, dB, dC, dz, dA, dD, ddt_bias, dconv_w, dconv_b, d_init_state,
//          d_init_conv_state, in that order.
// Every array lives in its own exact-size heap block, so any access outside it is reported by
// AddressSanitizer; outputs and workspace start as NaN bytes, so anything left unwritten shows.
#define SSD_EMU 1
#include "ssd_backward.cu"

#include <stdio.h>
#include <stdlib.h>

#include <memory>
#include <vector>

namespace {

struct Blob {
    std::unique_ptr<unsigned char[]> p;
    size_t n = 0;
};

Blob read_blob(FILE* f, size_t bytes) {
    Blob b;
    b.n = bytes;
    b.p.reset(new unsigned char[bytes ? bytes : 1]);
    if (bytes && fread(b.p.get(), 1, bytes, f) != bytes) {
        fprintf(stderr, "short input\n");
        exit(2);
    }
    return b;
}

Blob nan_blob(size_t bytes) {
    Blob b;
    b.n = bytes;
    b.p.reset(new unsigned char[bytes ? bytes : 1]);
    memset(b.p.get(), 0xFF, bytes ? bytes : 1);
    return b;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 3) {
        fprintf(stderr, "usage: run_backward in.bin out.bin\n");
        return 2;
    }
    FILE* f = fopen(argv[1], "rb");
    if (!f) return 2;
    int64_t hd[11];
    if (fread(hd, sizeof(int64_t), 11, f) != 11) return 2;
    const int64_t batch = hd[0], L = hd[1];
    const int H = (int)hd[2], P = (int)hd[3], N = (int)hd[4], G = (int)hd[5];
    const bool abf = hd[6] != 0, dbf = hd[7] != 0;
    const size_t HP = (size_t)H * P, GN = (size_t)G * N, conv_dim = HP + 2 * GN;
    const size_t ae = abf ? 2 : 4, de = dbf ? 2 : 4, rows = (size_t)(batch * L);

    Blob A = read_blob(f, H * 4), D = read_blob(f, H * 4), dtb = read_blob(f, H * 4);
    Blob cw = read_blob(f, conv_dim * 16), cb = read_blob(f, conv_dim * 4);
    Blob x = read_blob(f, rows * HP * ae), dt = read_blob(f, rows * H * ae), Bm = read_blob(f, rows * GN * ae),
         Cm = read_blob(f, rows * GN * ae), z = read_blob(f, rows * HP * ae), dy = read_blob(f, rows * HP * de);
    const size_t state = (size_t)batch * H * P * N;
    Blob is, ics, dfin;
    if (hd[8]) is = read_blob(f, state * 4);
    if (hd[9]) ics = read_blob(f, (size_t)batch * conv_dim * 3 * ae);
    if (hd[10]) dfin = read_blob(f, state * 4);
    fclose(f);

    Blob o_dx = nan_blob(rows * HP * 4), o_ddt = nan_blob(rows * H * 4), o_dB = nan_blob(rows * GN * 4),
         o_dC = nan_blob(rows * GN * 4), o_dz = nan_blob(rows * HP * 4), o_dA = nan_blob(H * 4),
         o_dD = nan_blob(H * 4), o_dtb = nan_blob(H * 4), o_cw = nan_blob(conv_dim * 16), o_cb = nan_blob(conv_dim * 4),
         o_is = nan_blob(state * 4), o_ics = nan_blob((size_t)batch * conv_dim * 3 * 4);
    Blob ws = nan_blob(ssd::bwd::workspace_bytes(batch, L, H, P, N, G));

    ssd::bwd::BwdArgs a{};
    a.batch = batch;
    a.L = L;
    a.H = H;
    a.P = P;
    a.N = N;
    a.G = G;
    a.act_bf16 = abf;
    a.dy_bf16 = dbf;
    a.A = (const float*)A.p.get();
    a.D = (const float*)D.p.get();
    a.dt_bias = (const float*)dtb.p.get();
    a.conv_w = (const float*)cw.p.get();
    a.conv_b = (const float*)cb.p.get();
    a.x = x.p.get();
    a.dt = dt.p.get();
    a.B = Bm.p.get();
    a.C = Cm.p.get();
    a.z = z.p.get();
    a.dy = dy.p.get();
    a.init_state = hd[8] ? (const float*)is.p.get() : nullptr;
    a.init_conv_state = hd[9] ? ics.p.get() : nullptr;
    a.d_final = hd[10] ? (const float*)dfin.p.get() : nullptr;
    a.dx = (float*)o_dx.p.get();
    a.ddt = (float*)o_ddt.p.get();
    a.dB = (float*)o_dB.p.get();
    a.dC = (float*)o_dC.p.get();
    a.dz = (float*)o_dz.p.get();
    a.dA = (float*)o_dA.p.get();
    a.dD = (float*)o_dD.p.get();
    a.ddt_bias = (float*)o_dtb.p.get();
    a.dconv_w = (float*)o_cw.p.get();
    a.dconv_b = (float*)o_cb.p.get();
    a.d_init_state = (float*)o_is.p.get();
    a.d_init_conv_state = (float*)o_ics.p.get();
    a.workspace = ws.p.get();
    if (ssd::bwd::launch_prefill_backward(a, nullptr) != cudaSuccess) return 3;

    FILE* o = fopen(argv[2], "wb");
    if (!o) return 2;
    for (const Blob* b : {&o_dx, &o_ddt, &o_dB, &o_dC, &o_dz, &o_dA, &o_dD, &o_dtb, &o_cw, &o_cb, &o_is, &o_ics})
        if (b->n) fwrite(b->p.get(), 1, b->n, o);
    fclose(o);
    return 0;
}
