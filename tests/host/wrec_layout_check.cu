// Host-side check of the folded weight record layout shared by the fold
// writers (fold_kernel, fold_unit) and the score loops (score_core.cuh and
// the pipelined kernel's slice loop).  Built with nvcc and run on the CPU: it
// only evaluates the constexpr index helpers, no device code runs.
//
// The score loops read, per head and 16-byte key chunk c (bands 4c..4c+3),
// three float4 words of the record: (ReA_4c, ReA_4c+1, ImA_4c, ImA_4c+1),
// (ReA_4c+2, ReA_4c+3, ImA_4c+2, ImA_4c+3) and (c_4c, ..., c_4c+3); the
// float32 loop reads, for half h of the chunk, the float4 at 4h and the
// float2 at 8 + 2h.  Prints "ok" and exits 0 when every band's slots are
// where those reads expect them and the 3 x 64 slots tile the record.
#include <cstdio>

#include "../../rope_aware_kv_b200/csrc/tri_internal.cuh"

using namespace tri;

int main() {
    int used[kWHead] = {0};
    int bad = 0;
    auto expect = [&](bool ok, const char* what, int f) {
        if (!ok) {
            std::printf("band %d: %s\n", f, what);
            ++bad;
        }
    };
    for (int f = 0; f < kF; ++f) {
        const int base = (f >> 2) * kWChunk, i = f & 3;
        const int re = wrec_re(f), im = wrec_im(f), c = wrec_c(f);
        for (int s : {re, im, c}) {
            expect(s >= 0 && s < kWHead, "slot outside the head record", f);
            if (s >= 0 && s < kWHead) ++used[s];
        }
        // bf16 loop: word i >> 1 holds (Re, Re, Im, Im) of bands 2(i >> 1), +1.
        expect(re == base + 4 * (i >> 1) + (i & 1), "real part not where the bf16 loop reads it", f);
        expect(im == base + 4 * (i >> 1) + 2 + (i & 1), "imaginary part misplaced", f);
        expect(c == base + 8 + i, "norm weight misplaced", f);
        // float32 loop: half h = i >> 1 reads the float4 at 4h and the float2 at 8 + 2h.
        const int h = i >> 1;
        expect(re - base - 4 * h == (i & 1), "float32 loop: real part", f);
        expect(im - base - 4 * h == 2 + (i & 1), "float32 loop: imaginary part", f);
        expect(c - base - 8 - 2 * h == (i & 1), "float32 loop: norm weight", f);
    }
    for (int s = 0; s < kWHead; ++s)
        if (used[s] != 1) {
            std::printf("slot %d used %d times\n", s, used[s]);
            ++bad;
        }
    if (bad) return 1;
    std::printf("ok\n");
    return 0;
}
