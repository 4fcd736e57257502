// Host-side checks of the kernels' planning arithmetic, compiled from the
// library's own headers and run on the CPU (tests/test_host_plans.py): the unit
// split of the decode kernels, the per-layer rotation of the persistent stack,
// its per-buffer count targets, the shared-memory layouts against the per-block
// limit, the router's K splits, the B-fragment word order, and the NVFP4 tile
// images (every byte of a stage written once, a row's scale factors of one
// k-block in one word, the gate/up row order).  Prints "ok" or
// the first failed check, and exits nonzero on a failure.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../fp4_expert_gemv_b200/csrc/router.cuh"
#include "../fp4_expert_gemv_b200/csrc/stack_decode.cuh"
#include "../fp4_expert_gemv_b200/csrc/nvfp4.cuh"
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
    // NVFP4 tile images: code bytes, A and B scale factors each a bijection onto their region
    {
        std::vector<int> seen(fe::kNvBChunk, 0);
        for (int r = 0; r < fe::kNvN; ++r)
            for (int kb = 0; kb < 128; ++kb) ++seen[fe::nv_code_off(r, kb)];
        for (int n = 0; n < fe::kNvN; ++n)
            for (int j = 0; j < 16; ++j) ++seen[fe::nv_sfb_off(n, j)];
        for (uint32_t i = 0; i < fe::kNvBChunk; ++i) CHECK(seen[i] == 1, "B image byte %u seen %d", i, seen[i]);
        std::vector<int> sa(fe::kNvAChunk, 0);
        for (int r = 0; r < fe::kNvM; ++r) {
            for (int kb = 0; kb < 128; ++kb) ++sa[fe::nv_code_off(r, kb)];
            for (int j = 0; j < 16; ++j) ++sa[fe::nv_sfa_off(r, j)];
        }
        for (uint32_t i = 0; i < fe::kNvAChunk; ++i) CHECK(sa[i] == 1, "A image byte %u seen %d", i, sa[i]);
        // a row's scale factors of one k-block are one 32-bit word (the tensor core reads them as one)
        for (int r = 0; r < fe::kNvN; ++r)
            for (int q = 0; q < 4; ++q) {
                CHECK(fe::nv_sfb_off(r, 4 * q) % 4 == 0 && fe::nv_sfb_off(r, 4 * q + 3) == fe::nv_sfb_off(r, 4 * q) + 3,
                      "B row %d k-block %d", r, q);
                if (r < fe::kNvM)
                    CHECK(fe::nv_sfa_off(r, 4 * q) % 4 == 0 && fe::nv_sfa_off(r, 4 * q + 3) == fe::nv_sfa_off(r, 4 * q) + 3,
                          "A row %d k-block %d", r, q);
            }
        for (int I : {128, 256, 768}) {
            std::vector<int> col(2 * I, 0);
            for (int R = 0; R < 2 * I; ++R) ++col[fe::nv_gate_up_column(R, I)];
            for (int n = 0; n < 2 * I; ++n) CHECK(col[n] == 1, "I=%d column %d", I, n);
            // gate and up of act column i sit 16 rows apart in one 32-row group
            for (int i = 0; i < I; ++i) {
                const int Rg = 32 * (i / 16) + i % 16;
                CHECK(fe::nv_gate_up_column(Rg, I) == i && fe::nv_gate_up_column(Rg + 16, I) == I + i, "I=%d i=%d", I, i);
            }
        }
        // the scale-factor layout of CUTLASS's sm100 block-scaled K-major atom: per 128 rows and
        // 4 factors (one 64-wide k-block), shape ((32, 4), (16, 4)) with strides ((16, 4), (0, 1))
        // over (row, k); further 128-row blocks 512 bytes apart, k-blocks after all rows' blocks
        for (int n = 0; n < fe::kNvN; ++n)
            for (int k = 0; k < fe::kNvKc; ++k) {
                const int q = k / 64, kk = k % 64, nb = n / 128, m = n % 128;
                const uint32_t atom = 16u * (m % 32) + 4u * (m / 32) + 0u * (kk % 16) + 1u * (kk / 16);
                CHECK(fe::nv_sfb_off(n, k / 16) == fe::kNvBCodes + 1024u * q + 512u * nb + atom, "B n=%d k=%d", n, k);
                if (n < fe::kNvM)
                    CHECK(fe::nv_sfa_off(n, k / 16) == fe::kNvACodes + 512u * q + atom, "A n=%d k=%d", n, k);
            }
        CHECK(fe::nv_smem_bytes() <= kMaxSmem, "NVFP4 tiles %u", fe::nv_smem_bytes());
        CHECK(256u + 4u * fe::kNvSfCols <= fe::kNvTmemCols, "TMEM columns");
        CHECK(fe::nv_instr_desc(256) == ((1u << 7) | (1u << 10) | (32u << 17) | (8u << 24)), "instruction descriptor");
    }
    if (failures) {
        std::printf("%d checks failed\n", failures);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
