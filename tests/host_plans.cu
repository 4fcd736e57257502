// Host-side checks of the kernels' planning arithmetic, compiled from the
// library's own headers and run on the CPU (tests/test_host_plans.py): the unit
// split of the decode kernels, the per-layer rotation of the persistent stack,
// its per-buffer count targets, the shared-memory layouts against the per-block
// limit, the router's K splits, and the B-fragment word order.  Prints "ok" or
// the first failed check, and exits nonzero on a failure.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../fp4_expert_gemv_b200/csrc/router.cuh"
#include "../fp4_expert_gemv_b200/csrc/stack_decode.cuh"
#include "../fp4_expert_gemv_b200/csrc/tcgen05.cuh"

static int failures = 0;
#define CHECK(cond, ...)                                        \
    do {                                                        \
        if (!(cond)) {                                          \
            if (failures++ < 10) {                              \
                std::printf("FAILED %s: ", #cond);              \
                std::printf(__VA_ARGS__);                       \
                std::printf("\n");                              \
            }                                                   \
        }                                                       \
    } while (0)

constexpr uint32_t kMaxSmem = 232448;   // dynamic shared memory a block may opt into

int main()
{
    // unit split: CTA c takes [first(c), first(c + 1)); a partition, shares differ by at most one
    for (int G : {132, 148, 160})
        for (int U = 0; U <= 3000; U += 7) {
            CHECK(fe::dec_unit_first(0, U, G) == 0 && fe::dec_unit_first(G, U, G) == U, "G=%d U=%d", G, U);
            for (int c = 0; c < G; ++c) {
                const int n = fe::dec_unit_first(c + 1, U, G) - fe::dec_unit_first(c, U, G);
                CHECK(n == U / G || n == (U + G - 1) / G, "G=%d U=%d c=%d n=%d", G, U, c, n);
            }
        }
    // the stack's rotation: for every layer, CTA c -> share (c + 53 l) mod G is a permutation
    for (int G : {132, 148, 160})
        for (int l = 0; l < fe::kStkMaxLayers; ++l) {
            std::vector<int> seen(G, 0);
            for (int c = 0; c < G; ++c) ++seen[(c + l * fe::kStkRotate) % G];
            for (int v = 0; v < G; ++v) CHECK(seen[v] == 1, "G=%d l=%d v=%d", G, l, v);
        }
    // per-buffer count targets: the events of every layer of buffer l % kStkBufs up to l in
    // this launch and all layers of that buffer in the launches before
    for (int L : {1, 2, 5, 6, 7, 13, 48, 64})
        for (unsigned long long epoch = 0; epoch < 4; ++epoch)
            for (int l = 0; l < L; ++l)
                for (int per : {1, 16, 128, 148}) {
                    unsigned long long brute = 0;
                    const int b = l % fe::kStkBufs;
                    for (unsigned long long e = 0; e <= epoch; ++e)
                        for (int m = 0; m < L; ++m)
                            if (m % fe::kStkBufs == b && (e < epoch || m <= l)) brute += (unsigned long long)per;
                    CHECK(fe::stack_count_through(epoch, L, l, per) == brute, "L=%d epoch=%llu l=%d per=%d", L, epoch,
                          l, per);
                }
    // launch tags differ for different (launch, layer)
    for (int L : {1, 48})
        for (unsigned long long e = 0; e < 3; ++e)
            for (int l = 0; l < L; ++l)
                CHECK(fe::stack_tag(e, L, l) != 0 && (l == 0 || fe::stack_tag(e, L, l) != fe::stack_tag(e, L, l - 1)),
                      "L=%d e=%llu l=%d", L, e, l);
    // shared memory of the persistent stack: fits, regions in order and aligned
    for (int H = 64; H <= fe::kDecMaxH; H += 64) {
        const fe::StackSmem s = fe::stack_smem_layout(H);
        CHECK(s.total <= kMaxSmem, "H=%d total=%u", H, s.total);
        CHECK(s.mbar < s.shared && s.shared < s.red && s.red < s.land && s.land < s.xs && s.xs < s.xr &&
                  s.xr < s.total,
              "H=%d order", H);
        CHECK(s.land % 16 == 0 && s.xr % 16 == 0 && s.mbar % 8 == 0, "H=%d alignment", H);
        CHECK(s.xs >= s.land + (uint32_t)fe::kDecMaxCtas * fe::kStkLandRow, "H=%d landing rows", H);
        // an INT2 unit fits an E2M1 slot of the single-launch kernel
        CHECK(2 * fe::int2_block_bytes(H) <= 2 * fe::block_bytes(H), "H=%d", H);
    }
    CHECK(fe::tc_smem_bytes() <= kMaxSmem, "tensor-core tiles %u", fe::tc_smem_bytes());
    // router K splits: a power of two up to 8 that divides the 64-wide chunks of H, its
    // partials within the reserved space
    for (int H : {64, 192, 256, 512, 2048})
        for (int E : {8, 40, 128, 512})
            for (int T = 1; T <= 300; ++T) {
                const int ks = fe::router_splits(T, H, E);
                CHECK(ks >= 1 && ks <= fe::kRtMaxSplits && (ks & (ks - 1)) == 0, "T=%d H=%d E=%d ks=%d", T, H, E, ks);
                CHECK((H / 64) % ks == 0, "T=%d H=%d E=%d ks=%d", T, H, E, ks);
                CHECK(ks == 1 || (long long)ks * T * E <= fe::kRtSplitFloats, "T=%d H=%d E=%d ks=%d", T, H, E, ks);
            }
    // B fragment order: a permutation of each block of 32 words
    for (uint32_t base = 0; base < 1024; base += 32) {
        std::vector<int> seen(32, 0);
        for (uint32_t kp = base; kp < base + 32; ++kp) {
            const uint32_t w = fe::bfrag_word(kp);
            CHECK(w >= base && w < base + 32, "kp=%u w=%u", kp, w);
            if (w >= base && w < base + 32) ++seen[w - base];
        }
        for (int i = 0; i < 32; ++i) CHECK(seen[i] == 1, "block %u word %d", base, i);
    }
    if (failures) {
        std::printf("%d checks failed\n", failures);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
