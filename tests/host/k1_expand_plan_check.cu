// k1_expand_plan_check.cu -- host-side check of how K1 shares out the weight
// expansion it runs beside the rows (kFlExpand), using the kernel header's own
// launch configuration (Cfg) and routing rule (expand_rides_along_l).  With the
// grid the launcher picks, group g of the ng groups widens chunk rg at each of
// its row groups rg = g, g + ng, ... (those below M's row groups), then the
// chunk where its rows stop and every ng-th one after it.  For each shape it
// checks that
//   1. the chunks are whole (W x 4 words each, dividing N K / 16 words),
//   2. every chunk is widened exactly once,
//   3. the routing rule takes the expansion into K1 exactly for the shapes
//      expected (the ones the GPU tests and the benchmark run through it),
// and prints one line per shape; and that the word widening both expansion
// paths share (expand_ternary_word) gives byte 4i + b = the two-bit field at
// bits 8b + 2i minus one (mod 256) for every low and high half-word, so no
// borrow crosses a byte.  Exits non-zero on any failure.
#include <cstdio>
#include <vector>

#include "k1_impl.cuh"

using namespace hbl::k1;

template <int L, int RL>
static int cover(long long M, int N, int sms, int* tail_max) {
    using C = Cfg<L, RL>;
    const long long groups = (M + C::kRowsPerGroup - 1) / C::kRowsPerGroup;
    long long ctas = (groups + C::kGroupsPerCta - 1) / C::kGroupsPerCta;
    if (ctas > (long long)sms * C::kMinBlocks) ctas = (long long)sms * C::kMinBlocks;
    if (ctas < 1) ctas = 1;
    const long long ng = ctas * C::kGroupsPerCta;
    const long long words = (long long)N * (C::K / 16);
    const long long chunk = (long long)C::W * 4;
    if (words % chunk != 0) return 1;
    const long long chunks = words / chunk;
    std::vector<int> seen(chunks, 0);
    *tail_max = 0;
    for (long long g = 0; g < ng; ++g) {
        long long rg = g;
        for (; rg < groups; rg += ng)
            if (rg < chunks) ++seen[rg];
        int tail = 0;
        for (long long c = rg; c < chunks; c += ng, ++tail) ++seen[c];
        if (tail > *tail_max) *tail_max = tail;
    }
    int bad = 0;
    for (long long c = 0; c < chunks; ++c) bad += seen[c] != 1;
    return bad;
}

template <int L>
static int check(long long M, int N, int expect_fused) {
    const int sms = 148;
    int tail = 0;
    const int bad = (L == 14 && M <= (long long)sms * Cfg<L>::kMinBlocks)
                        ? cover<L, 6>(M, N, sms, &tail)
                        : cover<L, reg_log(L)>(M, N, sms, &tail);
    const bool fused = expand_rides_along_l<L>(M, N, sms);
    const bool ok = bad == 0 && (expect_fused < 0 || fused == (expect_fused != 0));
    printf("K=%d M=%lld N=%d: in K1 %d, chunks after the rows <= %d: %s\n", 1 << L, M, N,
           (int)fused, tail, ok ? "ok" : "FAIL");
    return ok ? 0 : 1;
}

// expand_ternary_word against the packing's definition (weight j of a word at
// bits 8(j%4) + 2(j/4), code t + 1), for words w = lo | hi << 16.
static int check_widening() {
    int bad = 0;
    auto one = [&](uint32_t w) {
        const uint4 v = hbl::expand_ternary_word(w);
        const uint32_t part[4] = {v.x, v.y, v.z, v.w};
        for (int i = 0; i < 4; ++i)
            for (int b = 0; b < 4; ++b) {
                const uint32_t code = (w >> (8 * b + 2 * i)) & 3u;
                const uint32_t want = (code + 255u) & 255u;  // code - 1 mod 256
                if (((part[i] >> (8 * b)) & 255u) != want) ++bad;
            }
    };
    const uint32_t others[] = {0x0000u, 0xffffu, 0x5555u, 0xaaaau, 0x1234u};
    for (uint32_t h = 0; h < 65536u; ++h)
        for (uint32_t o : others) {
            one(h | (o << 16));
            one(o | (h << 16));
        }
    printf("word widening, %d half-word patterns x %d: %s\n", 65536, 2 * 5, bad ? "FAIL" : "ok");
    return bad ? 1 : 0;
}

int main() {
    int bad = check_widening();
    // taken into K1: the benchmark's W_down and the GPU test shapes
    bad += check<14>(8192, 4096, 1);
    bad += check<12>(8192, 4096, 1);
    bad += check<7>(257, 16, 1);
    bad += check<12>(1777, 2048, 1);
    bad += check<14>(445, 656, 1);
    bad += check<13>(600, 1200, 1);
    // left to the separate kernel: most chunks would come after the rows
    bad += check<14>(2048, 4096, 0);
    bad += check<14>(300, 4096, 0);
    bad += check<12>(8192, 11008, 0);
    bad += check<11>(300, 4000, 0);
    // coverage alone, over a spread of shapes (the kernel is correct either way)
    const long long Ms[] = {1, 31, 257, 444, 445, 1000, 4099};
    const int Ns[] = {16, 272, 4000, 11008};
    for (long long M : Ms)
        for (int N : Ns) {
            bad += check<8>(M, N, -1);
            bad += check<11>(M, N, -1);
            bad += check<14>(M, N, -1);
            bad += check<15>(M, N, -1);
        }
    return bad ? 1 : 0;
}
