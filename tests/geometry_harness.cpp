// Host build of the kernels' geometry and scheduling headers: dumps the token
// slot map, the TMA box origins and the (query tile, key tile) pairs that the
// forward and backward work items visit, for checking on the CPU.
#include <cstdio>
#include <cstdlib>

#include "geometry.cuh"
#include "schedule.cuh"

using namespace fswin;

// Division by invariant integers against the hardware divide: small and large
// divisors, numerators near multiples of the divisor and near 2^31.
static int check_fastdiv() {
    unsigned long long bad = 0, n_checked = 0;
    const uint32_t ds[] = {1u, 2u, 3u, 5u, 7u, 9u, 16u, 48u, 64u, 100u, 255u, 256u, 1000u, 4096u, 6553u, 65535u,
                           65536u, 123457u, 1u << 20, (1u << 20) + 1u, 33554431u, 1u << 30, (1u << 31) - 1u, 1u << 31};
    for (uint32_t d : ds) {
        const FastDiv f = make_fastdiv(d);
        for (uint32_t k = 0; k < 2000; ++k) {
            const uint32_t cand[] = {k, k * d, k * d - 1u, k * d + 1u, 0x7FFFFFFFu - k, 0x80000000u - k,
                                     static_cast<uint32_t>((k * 2654435761ull) & 0x7FFFFFFFu)};
            for (uint32_t n : cand) {
                if (n > 0x80000000u) continue;
                ++n_checked;
                if (fdiv(f, n) != n / d) ++bad;
            }
        }
    }
    std::printf("D %llu %llu\n", n_checked, bad);
    return bad ? 1 : 0;
}

int main(int argc, char** argv) {
    if (argc == 2 && argv[1][0] == 'D') return check_fastdiv();
    if (argc != 8) return 1;
    int a[7];
    for (int i = 0; i < 7; ++i) a[i] = std::atoi(argv[i + 1]);
    Geo g;
    if (geo_init(&g, a[0], a[1], a[2], a[3], a[4], a[5], a[6])) {
        std::printf("REJECT\n");
        return 0;
    }
    std::printf("G %d %d %d %lld %d %d %d %d %d\n", g.N, g.BT, g.bpt, g.tiles, g.tpw, g.bh, g.bw, g.Hp, g.Wp);
    for (long long t = 0; t < g.tiles; ++t)
        for (int p = 0; p < kTile; ++p) {
            const Slot s = slot_of(g, t, p);
            std::printf("S %lld %d %d %d %d %d %d %lld %d %d\n", t * kTile + p, s.box.b, s.row, s.col, s.i, s.j,
                        s.box.label, s.box.gw, s.box.valid ? 1 : 0, s.valid ? 1 : 0);
        }
    for (long long b = 0; b < g.tiles * g.bpt; ++b) {
        const Box x = box_of(g, b);
        std::printf("X %lld %d %d %d %d\n", b, x.b, x.row0, x.col0, x.valid ? 1 : 0);
    }
    for (long long it = 0; it < fwd_item_count(g); ++it) {
        const FwdItem I = fwd_item(g, it);
        for (int u = 0; u < I.nkv; ++u)
            if ((I.act >> u) & 1u) std::printf("F %lld %d %lld %lld\n", it, I.h, I.X, I.kv0 + u);
    }
    for (long long it = 0; it < bwd_item_count(g); ++it) {
        const BwdItem I = bwd_item(g, it);
        for (int n = 0; n < I.nq; ++n)
            if (bwd_active(g, I, n)) std::printf("B %lld %d %lld %lld\n", it, I.h, I.u, I.q0 + n);
    }
    return 0;
}
