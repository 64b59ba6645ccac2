// k1_layout_check.cu -- host-side check of K1's register/thread layouts and
// shared-memory exchange addressing, using the kernel header's own constexpr
// layout functions (Cfg, Lay, swz).  For every (K, values per thread) the
// kernels instantiate it checks that
//   1. each layout maps (thread, register slot) one-to-one onto the row, and
//   2. every 16-byte exchange access (write in layout p - 1, read in layout p)
//      is free of bank conflicts: in each quarter-warp the eight chunk
//      addresses fall into eight different 16-byte bank groups,
// and that writer and reader address an element's chunk identically.
// Prints one line per configuration and exits non-zero on any failure.
#include <cstdio>
#include <vector>

#include "k1_impl.cuh"

using namespace hbl::k1;

template <int L, int RL>
static int check() {
    using C = Cfg<L, RL>;
    using Y = Lay<L, RL>;
    constexpr int K = C::K, R = C::R, W = C::W, T = C::T;
    int bad = 0;
    // element index of thread w (within its group) and register slot i in layout p
    auto thr_off = [&](int p, int w) {
        const int j = (T >= 32) ? w : ((w & 31) % T);
        const int rig = (T >= 32) ? 0 : ((w & 31) / T);
        int e = 0;
        for (int tb = 0; tb < C::t; ++tb) e |= ((j >> tb) & 1) << Y::thr_idx(p, tb);
        return e + rig * K;
    };
    const int P_LAST = C::kPasses;
    for (int p = 0; p <= P_LAST; ++p) {
        std::vector<int> seen(K * C::kRowsPerGroup, 0);
        for (int w = 0; w < W; ++w)
            for (int i = 0; i < R; ++i) {
                const int e = thr_off(p, w) | Y::reg_off(p, i);
                if (e < 0 || e >= K * C::kRowsPerGroup) { ++bad; continue; }
                ++seen[e];
            }
        for (int e = 0; e < K * C::kRowsPerGroup; ++e)
            if (seen[e] != 1) ++bad;
    }
    // exchanges: writer (layout p - 1) and reader (layout p), 16-byte chunk c
    for (int p = 1; p <= P_LAST; ++p)
        for (int side = 0; side < 2; ++side) {
            const int q = side == 0 ? p - 1 : p;
            for (int c = 0; c < R / 4; ++c) {
                for (int w0 = 0; w0 < W; w0 += 8) {  // quarter-warps
                    int groups = 0;
                    for (int l = 0; l < 8; ++l) {
                        const int w = w0 + l;
                        const unsigned tb = swz((unsigned)thr_off(q, w) >> 2);
                        const unsigned rc = swz((unsigned)Y::reg_off(q, 4 * c) >> 2);
                        const unsigned chunk = tb ^ rc;
                        // the chunk holds elements e .. e + 3 (index bits 0, 1 in registers)
                        const unsigned e = (unsigned)(thr_off(q, w) | Y::reg_off(q, 4 * c));
                        if (chunk != swz(e >> 2)) ++bad;
                        groups |= 1 << (chunk & 7);
                    }
                    if (groups != 0xFF) ++bad;
                }
            }
        }
    std::printf("K=%d values/thread=%d threads/row=%d exchanges=%d: %s\n", K, R, T, P_LAST,
                bad ? "FAIL" : "ok");
    return bad;
}

int main() {
    int bad = 0;
    // the plain kernel's shapes
    bad += check<7, reg_log(7)>();
    bad += check<8, reg_log(8)>();
    bad += check<9, reg_log(9)>();
    bad += check<10, reg_log(10)>();
    bad += check<11, reg_log(11)>();
    bad += check<12, reg_log(12)>();
    bad += check<13, reg_log(13)>();
    bad += check<14, reg_log(14)>();
    bad += check<15, reg_log(15)>();
    // 64 values per thread: the few-row launch at K = 16384 and the decode kernels
    bad += check<12, 6>();
    bad += check<13, 6>();
    bad += check<14, 6>();
    return bad ? 1 : 0;
}
