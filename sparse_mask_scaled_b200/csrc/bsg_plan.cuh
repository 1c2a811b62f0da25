// Closed-form tile plan of a block + strided + global mask.
//
// The pattern (the "Sparse Attention" notes page, pattern list: block or
// strided patterns and global tokens): row i attends to key j when
//   block > 0 and i div block == j div block             (block-local)
//   S > 0 and (j - i) mod S == 0                          (strided)
//   i < ng or j < ng                                      (global tokens)
// When block divides 128, S is 0 or 128, ng <= 128, n is a multiple of 128 and
// the block or global part is present, every query block's tensor-core tiles
// and every tile's per-row bits follow from (n, block, S, ng) alone, so the
// forward pass needs no CSR and no stored plan:
//
// Regular query block qb (rows 128 qb + t, t < 128) takes the key tiles
//   qb        when block > 0   (block-local entries; j = i lies there too),
//   0         when ng > 0      (keys j < ng, and the strided key j = t),
//   all       when ng > 0 and qb == 0, but beyond tiles 0 and qb only for the
//             global rows t < ng (each attends to every key),
// and in those tiles every entry of the mask that the rule above assigns it.
//
// Strided entries elsewhere go to permuted blocks. With G = n / 128, write
// i = 128 k + r (residue r, position k); the strided keys of row i are
// j = 128 k' + r for every k'. In residue-permuted order (row i at r G + k)
// they form a G x G dense block per residue, cut into 128 x 128 tiles:
// permuted block (r, pqb) holds rows k = 128 pqb + t, its tile pkt keys
// k' = 128 pkt + c, and takes the strided entries the regular tiles do not
// hold: all (k, k') but k' == k (block > 0), k' == 0 (ng > 0), and none of a
// global row (i < ng).
//
// A row with entries in both kinds of block has two partial softmax states
// (running max, sum, weighted V sum) that are merged with the running-max /
// running-sum rule ("Implementing and Optimizing the Scaled Dot-Product
// Attention on Streaming Dataflow", proposed method).
//
// Everything here is plain integer arithmetic, usable on the host as well.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define BSG_HD __host__ __device__ __forceinline__
#else
#define BSG_HD inline
#endif

namespace spattn {
namespace bsg {

constexpr int kTile = 128;

// Bits of the columns [c0, c0 + 32) that lie in [lo, hi).
BSG_HD uint32_t run_word(int lo, int hi, int c0) {
    int a = lo - c0, z = hi - c0;
    a = a < 0 ? 0 : (a > 32 ? 32 : a);
    z = z < 0 ? 0 : (z > 32 ? 32 : z);
    if (z <= a) return 0u;
    const uint32_t top = z == 32 ? 0xffffffffu : ((1u << z) - 1u);
    return top & ~((1u << a) - 1u);
}

struct Shape {
    int n, block, S, ng;
    int nqb;            // 128-row query blocks (= key tiles)
    int G;              // positions per residue (n / 128) when S == 128, else 0
    int npqb;           // permuted blocks per residue (ceil(G / 128))
    int chunk_tiles;    // tiles per chunk of the global-row block
    int nch;            // chunks of query block 0 (1 unless ng > 0)
    int n_lead;         // chunk items at the head of each (b, h) item list
    int nreg;           // further regular items (query blocks 1.. or 0..)
    int nperm;          // permuted items (128 * npqb, or 0)
    int items_per_head;
};

// Whether the closed form covers the parameters.
BSG_HD bool supported(int n, int block, int S, int ng) {
    if (n <= 0 || n % kTile != 0) return false;
    if (block < 0 || S < 0 || ng < 0 || ng > kTile) return false;
    if (block > 0 && kTile % block != 0) return false;
    if (S != 0 && S != kTile) return false;
    return block > 0 || ng > 0;
}

BSG_HD Shape shape(int n, int block, int S, int ng, int chunk_tiles) {
    Shape s;
    s.n = n;
    s.block = block;
    s.S = S;
    s.ng = ng;
    s.nqb = n / kTile;
    s.G = S == kTile ? n / kTile : 0;
    s.npqb = s.G > 0 ? (s.G + kTile - 1) / kTile : 0;
    s.chunk_tiles = chunk_tiles;
    s.nch = ng > 0 ? (s.nqb + chunk_tiles - 1) / chunk_tiles : 1;
    s.n_lead = ng > 0 ? s.nch : 0;
    s.nreg = ng > 0 ? s.nqb - 1 : s.nqb;
    s.nperm = s.G > 0 ? kTile * s.npqb : 0;
    s.items_per_head = s.n_lead + s.nreg + s.nperm;
    return s;
}

// One unit of work: a regular query block (or one chunk of block 0's tiles),
// or a permuted block.
struct Item {
    int bh;
    int perm;   // 0 regular, 1 permuted
    int qb;     // regular: query block; permuted: residue r
    int pqb;    // permuted: block of positions within the residue
    int chunk;  // regular block 0 with ng > 0: chunk number, else 0
    int u0;     // first tile of the chunk in the block's tile list
    int T;      // tiles of this item
};

// Item x of all bh_count * items_per_head, in four phases over every (b, h):
//   1. the chunks of query block 0 but the first (items with many tiles and
//      no dependency: they start early, so that they do not end last),
//   2. the permuted blocks,
//   3. the first chunk of query block 0 (or query block 0 itself),
//   4. the remaining regular blocks (the items with the fewest tiles: they
//      fill the end evenly).
// Rows met by both kinds of block start their regular part from the permuted
// part's published state; with every permuted block ahead of every regular
// one, a regular block almost never waits for its rows' state, and items
// taken in this order never wait for a later one. (Interleaving the two kinds
// head by head keeps the published states in L2 but makes regular blocks wait
// for late permuted ones, which cost more on one B200: 0.39 against 0.34 ms
// on the 16-head n = 16384 workload.)
BSG_HD Item item(const Shape& s, int64_t x64, int bh_count) {
    // 32-bit arithmetic: callers keep bh_count * items_per_head below 2^31
    int x = (int)x64;
    Item it;
    it.perm = 0;
    it.qb = 0;
    it.pqb = 0;
    it.chunk = 0;
    it.u0 = 0;
    const int rest_chunks = s.n_lead > 1 ? s.n_lead - 1 : 0;
    const int p1 = bh_count * rest_chunks, p2 = bh_count * s.nperm, p3 = s.n_lead > 0 ? bh_count : 0;
    int j;  // chunk (phases 1 and 3), permuted block (2) or regular block (4) within the (b, h)
    if (x < p1) {
        it.bh = x / rest_chunks;
        j = 1 + (x - it.bh * rest_chunks);
    } else if ((x -= p1) < p2) {
        it.bh = x / s.nperm;
        it.perm = 1;
        j = x - it.bh * s.nperm;
    } else if ((x -= p2) < p3) {
        it.bh = x;
        j = 0;
    } else {
        x -= p3;
        it.bh = x / s.nreg;
        j = s.n_lead + (x - it.bh * s.nreg);
    }
    if (it.perm) {
        it.qb = j / s.npqb;
        it.pqb = j - it.qb * s.npqb;
        it.T = s.npqb;
        return it;
    }
    if (j < s.n_lead) {  // a chunk of query block 0 (a mask with global rows)
        it.chunk = j;
        it.u0 = j * s.chunk_tiles;
        const int rest = s.nqb - it.u0;
        it.T = rest < s.chunk_tiles ? rest : s.chunk_tiles;
        return it;
    }
    it.qb = j - s.n_lead + (s.ng > 0 ? 1 : 0);
    // tiles 0 (global keys) and qb (block); block 0 here only when ng == 0
    it.T = (s.ng > 0 ? 1 : 0) + (s.block > 0 ? 1 : 0);
    return it;
}

// Whether a regular item starts from the published state of its rows'
// permuted parts (the item that holds tile 0 of a query block, when the
// pattern has permuted blocks).
BSG_HD bool starts_from_perm(const Shape& s, const Item& it) {
    return s.G > 0 && !it.perm && it.chunk == 0;
}

// Key tile of the item's tile u: a key tile for regular items (ascending),
// a tile of positions k' for permuted ones.
BSG_HD int key_tile(const Shape& s, const Item& it, int u) {
    if (it.perm) return u;
    if (s.ng > 0 && it.qb == 0) return it.u0 + u;
    if (s.ng > 0) return u == 0 ? 0 : it.qb;
    return it.qb;
}

// Row t of the item as a row of the Q/out tensors, or -1 when it does not exist.
BSG_HD int row_of(const Shape& s, const Item& it, int t) {
    if (!it.perm) return it.qb * kTile + t;
    const int k = it.pqb * kTile + t;
    return k < s.G ? k * kTile + it.qb : -1;
}

// Whether row i also has entries in a permuted block.
BSG_HD bool has_perm(const Shape& s, int i) {
    if (s.G == 0 || i < s.ng) return false;
    const int k = i / kTile;
    const int excl = (s.block > 0 ? 1 : 0) + (s.ng > 0 ? 1 : 0) - (s.block > 0 && s.ng > 0 && k == 0 ? 1 : 0);
    return s.G > excl;
}

// The 128 bits (w[c / 32] bit c % 32 = column c) of row t of the item in its
// key tile kt.
BSG_HD void row_bits(const Shape& s, const Item& it, int kt, int t, uint32_t (&w)[4]) {
    w[0] = w[1] = w[2] = w[3] = 0u;
    if (it.perm) {
        const int k = it.pqb * kTile + t;
        const int i = k * kTile + it.qb;
        if (k >= s.G || i < s.ng) return;
        const int c_self = k - kt * kTile;  // column of k' == k in this tile, if any
        for (int q = 0; q < 4; ++q) {
            uint32_t v = run_word(0, s.G - kt * kTile, 32 * q);
            if (s.block > 0 && c_self >= 32 * q && c_self < 32 * q + 32) v &= ~(1u << (c_self - 32 * q));
            if (s.ng > 0 && kt == 0 && q == 0) v &= ~1u;
            w[q] = v;
        }
        return;
    }
    const int i = it.qb * kTile + t;
    if (i < s.ng) {  // a global row: every key
        w[0] = w[1] = w[2] = w[3] = 0xffffffffu;
        return;
    }
    if (s.ng > 0 && it.qb == 0 && kt != 0) return;  // beyond tile 0 only the global rows
    for (int q = 0; q < 4; ++q) {
        uint32_t v = 0u;
        if (s.block > 0 && kt == it.qb) {
            const int b0 = (i / s.block) * s.block - kt * kTile;
            v |= run_word(b0, b0 + s.block, 32 * q);
        }
        if (s.ng > 0 && kt == 0) v |= run_word(0, s.ng, 32 * q);
        if (s.S == kTile && t >= 32 * q && t < 32 * q + 32) v |= 1u << (t - 32 * q);
        w[q] = v;
    }
}

}  // namespace bsg
}  // namespace spattn
