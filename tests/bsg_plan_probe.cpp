// Test driver for the closed-form block + strided + global tile plan
// (sparse_mask_scaled_b200/csrc/bsg_plan.cuh), built for the host by
// tests/test_bsg_plan_cpu.py. For the parameters on the command line it walks
// the work items of five (b, h) heads, keeps those of head 1, and for every
// tile and every row's bits writes
// to stdout, as raw bytes: the n x n count of how many times each entry (i, j)
// is computed (uint8), the per-row "has entries in a permuted block" flag
// computed from the bits (uint8 [n]) and the one bsg::has_perm reports (uint8
// [n]). Exit status 2 when the parameters are outside the closed form, 6 when
// a regular item that starts from published states comes before one of its
// head's permuted items.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "bsg_plan.cuh"

using namespace spattn::bsg;

int main(int argc, char** argv) {
    if (argc != 6) return 1;
    const int n = atoi(argv[1]), block = atoi(argv[2]), S = atoi(argv[3]), ng = atoi(argv[4]),
              chunk = atoi(argv[5]);
    if (!supported(n, block, S, ng)) return 2;
    const Shape s = shape(n, block, S, ng, chunk);
    std::vector<uint8_t> cnt((size_t)n * n, 0), perm_rows(n, 0), has(n, 0);
    // every item of five (b, h) heads (the order interleaves heads), keeping head 1's
    const int heads = 5;
    std::vector<int64_t> last_perm(heads, -1), first_reg(heads, -1);
    for (int64_t x = 0; x < (int64_t)heads * s.items_per_head; ++x) {
        const Item it = item(s, x, heads);
        if (it.bh < 0 || it.bh >= heads) return 3;
        if (it.perm) last_perm[it.bh] = x;
        else if (starts_from_perm(s, it) && first_reg[it.bh] < 0) first_reg[it.bh] = x;
        if (it.bh != 1) continue;
        for (int u = 0; u < it.T; ++u) {
            const int kt = key_tile(s, it, u);
            for (int t = 0; t < kTile; ++t) {
                uint32_t w[4];
                row_bits(s, it, kt, t, w);
                const int i = row_of(s, it, t);
                for (int c = 0; c < kTile; ++c) {
                    if (!((w[c / 32] >> (c % 32)) & 1u)) continue;
                    if (i < 0 || i >= n) return 4;  // a bit on a row that does not exist
                    const int j = it.perm ? (kt * kTile + c) * kTile + it.qb : kt * kTile + c;
                    if (j < 0 || j >= n) return 5;
                    if (it.perm) perm_rows[i] = 1;
                    uint8_t& e = cnt[(size_t)i * n + j];
                    if (e < 255) ++e;
                }
            }
        }
    }
    for (int h = 0; h < heads; ++h)
        if (last_perm[h] >= 0 && first_reg[h] >= 0 && last_perm[h] > first_reg[h]) return 6;
    for (int i = 0; i < n; ++i) has[i] = has_perm(s, i) ? 1 : 0;
    fwrite(cnt.data(), 1, cnt.size(), stdout);
    fwrite(perm_rows.data(), 1, n, stdout);
    fwrite(has.data(), 1, n, stdout);
    return 0;
}
