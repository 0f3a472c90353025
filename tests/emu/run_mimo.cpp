// run_mimo.cpp -- runs the MIMO decode kernel of ssd_mimo.cu on the CPU through the host emulation
// in emu_cuda.h (built with AddressSanitizer by the tests; never part of the library).
//
// usage: run_mimo <in.bin> <out.bin>
// in.bin:  9 int64 (batch, H, P, N, G, R, act_bf16, y_bf16, steps), then A, D, dt_bias [H] f32 and
//          the initial state [batch][H][P][N] f32, then per step x [batch][H][R][P], dt [batch][H],
//          B [batch][G][R][N], C [batch][G][R][N], z [batch][H][R][P] (activation dtype).
// out.bin: per step y [batch][H][R][P] (y dtype), then the final state (f32).
// Every array lives in its own exact-size heap block (AddressSanitizer reports any access outside
// it); y starts as NaN bytes, so anything left unwritten shows.
#define SSD_EMU 1
#include "ssd_mimo.cu"

#include <stdio.h>
#include <stdlib.h>

#include <memory>
#include <vector>

namespace {

std::unique_ptr<unsigned char[]> read_blob(FILE* f, size_t bytes) {
    std::unique_ptr<unsigned char[]> p(new unsigned char[bytes ? bytes : 1]);
    if (bytes && fread(p.get(), 1, bytes, f) != bytes) {
        fprintf(stderr, "short input\n");
        exit(2);
    }
    return p;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 3) return 2;
    FILE* f = fopen(argv[1], "rb");
    if (!f) return 2;
    int64_t hd[9];
    if (fread(hd, sizeof(int64_t), 9, f) != 9) return 2;
    const int64_t batch = hd[0], steps = hd[8];
    const int H = (int)hd[1], P = (int)hd[2], N = (int)hd[3], G = (int)hd[4], R = (int)hd[5];
    const bool abf = hd[6] != 0, ybf = hd[7] != 0;
    const size_t ae = abf ? 2 : 4, ye = ybf ? 2 : 4;
    const size_t nx = (size_t)batch * H * R * P, nb = (size_t)batch * G * R * N, nst = (size_t)batch * H * P * N;
    auto A = read_blob(f, H * 4), D = read_blob(f, H * 4), dtb = read_blob(f, H * 4);
    auto state = read_blob(f, nst * 4);
    FILE* o = fopen(argv[2], "wb");
    if (!o) return 2;
    for (int64_t s = 0; s < steps; ++s) {
        auto x = read_blob(f, nx * ae), dt = read_blob(f, (size_t)batch * H * ae), Bm = read_blob(f, nb * ae),
             Cm = read_blob(f, nb * ae), z = read_blob(f, nx * ae);
        std::unique_ptr<unsigned char[]> y(new unsigned char[nx * ye]);
        memset(y.get(), 0xFF, nx * ye);
        ssd::mimo::MimoArgs a{};
        a.batch = batch;
        a.H = H;
        a.P = P;
        a.N = N;
        a.G = G;
        a.R = R;
        a.act_bf16 = abf;
        a.y_bf16 = ybf;
        a.A = (const float*)A.get();
        a.D = (const float*)D.get();
        a.dt_bias = (const float*)dtb.get();
        a.x = x.get();
        a.dt = dt.get();
        a.B = Bm.get();
        a.C = Cm.get();
        a.z = z.get();
        a.ssm_state = (float*)state.get();
        a.y = y.get();
        if (ssd::mimo::launch_mimo_decode(a, nullptr) != cudaSuccess) return 3;
        fwrite(y.get(), 1, nx * ye, o);
    }
    fclose(f);
    fwrite(state.get(), 1, nst * 4, o);
    fclose(o);
    return 0;
}
