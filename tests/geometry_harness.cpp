// Host build of the kernels' geometry and scheduling headers: dumps the token
// slot map, the TMA box origins and the (query tile, key tile) pairs that the
// forward and backward work items visit, for checking on the CPU.
#include <cstdio>
#include <cstdlib>

#include "geometry.cuh"
#include "schedule.cuh"

using namespace fswin;

int main(int argc, char** argv) {
    if (argc != 8) return 1;
    int a[7];
    for (int i = 0; i < 7; ++i) a[i] = std::atoi(argv[i + 1]);
    Geo g;
    if (geo_init(&g, a[0], a[1], a[2], a[3], a[4], a[5], a[6])) {
        std::printf("REJECT\n");
        return 0;
    }
    std::printf("G %d %d %d %lld %d %d %d\n", g.N, g.BT, g.bpt, g.tiles, g.tpw, g.bh, g.bw);
    for (long long t = 0; t < g.tiles; ++t)
        for (int p = 0; p < kTile; ++p) {
            const Slot s = slot_of(g, t, p);
            std::printf("S %lld %d %d %d %d %d %d %lld %d\n", t * kTile + p, s.box.b, s.row, s.col, s.i, s.j,
                        s.box.label, s.box.gw, s.box.valid ? 1 : 0);
        }
    for (long long b = 0; b < g.tiles * g.bpt; ++b) {
        const Box x = box_of(g, b);
        std::printf("X %lld %d %d %d %d\n", b, x.b, x.row0, x.col0, x.valid ? 1 : 0);
    }
    for (long long it = 0; it < fwd_item_count(g); ++it) {
        const FwdItem I = fwd_item(g, it);
        for (int T = 0; T < 2; ++T) {
            const long long qt = T ? I.tB : I.tA;
            if (qt < 0) continue;
            for (int u = 0; u < I.nkv; ++u)
                if (fwd_active(g, I, T, u)) std::printf("F %lld %d %lld %lld\n", it, I.h, qt, I.kv0 + u);
        }
    }
    for (long long it = 0; it < bwd_item_count(g); ++it) {
        const BwdItem I = bwd_item(g, it);
        for (int n = 0; n < I.nq; ++n)
            if (bwd_active(g, I, n)) std::printf("B %lld %d %lld %lld\n", it, I.h, I.u, I.q0 + n);
    }
    return 0;
}
