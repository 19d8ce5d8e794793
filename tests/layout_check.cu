// Host-only check of the layout arithmetic the kernels share with the host
// (no kernels, no GPU): prints "ok" or the first violation and exits non-zero.
//
// TiledMatrix (quantize.cuh), compact form: for every (row n, 32-block b) of a matrix, the
// code slot (16 bytes) and the scale byte lie inside the expert's bytes, inside
// the chunk that chunk_offset / chunk_bytes give for (n / 128, b / 4), and no
// two (n, b) share a code slot or a scale byte; the chunks of an expert tile it
// with no gap (atom padding included) up to expert_bytes.
// sf_atom_offset (mxq.cuh): byte 16 (n % 32) + 4 ((n / 32) % 4) + q of atom
// n / 128, and a bijection from (row n < 256, block q < 4) onto the 1024
// bytes of two atoms.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../mxfp4_expert_gemm_router_b200/csrc/mxq.cuh"
#include "../mxfp4_expert_gemm_router_b200/csrc/quantize.cuh"

using namespace moe;

static int fail(const char* what, int a, int b, int c) {
    std::printf("FAIL %s (%d, %d, %d)\n", what, a, b, c);
    return 1;
}

static int check_matrix(int N, int K, int NM) {
    for (int sub = 0; sub < NM; ++sub) {
        TiledMatrix M{nullptr, N, K, NM, sub};
        const size_t total = M.expert_bytes();
        std::vector<unsigned char> code_used(total, 0), scale_used(total, 0);
        for (int n = 0; n < N; ++n)
            for (int b = 0; b < M.nb(); ++b) {
                size_t co, so;
                M.locate(n, b, co, so);
                const int ft = n / 128, rf = (N - 128 * ft) < 128 ? N - 128 * ft : 128, c = b / 4;
                const size_t c0 = M.chunk_offset(ft, c, rf), c1 = c0 + M.chunk_bytes(c, rf);
                if (co + 16 > total || so >= total) return fail("slot outside the expert", N, n, b);
                if (co < c0 || co + 16 > c1 || so < c0 || so >= c1) return fail("slot outside its chunk", N, n, b);
                for (int i = 0; i < 16; ++i)
                    if (code_used[co + i]++) return fail("code bytes shared", N, n, b);
                if (scale_used[so]++) return fail("scale byte shared", N, n, b);
                if (code_used[so] || scale_used[co]) return fail("code and scale overlap", N, n, b);
            }
    }
    // chunks tile the expert contiguously
    TiledMatrix M{nullptr, N, K, NM, 0};
    size_t expect = 0;
    for (int ft = 0; ft < M.tiles(); ++ft) {
        const int rf = (N - 128 * ft) < 128 ? N - 128 * ft : 128;
        if (M.tile_offset(ft) != expect) return fail("tile offset", N, K, ft);
        for (int c = 0; c < M.chunks(); ++c) {
            if (M.chunk_offset(ft, c, rf) != expect) return fail("chunk offset", N, ft, c);
            expect += M.chunk_bytes(c, rf);
        }
    }
    if (expect != M.expert_bytes()) return fail("expert bytes", N, K, NM);
    return 0;
}

// The padded form (layers with two-MXFP8-term operands): every part of a chunk
// is PAD_MAT bytes, codes [128 rows][64 B] then the atom, so that the tensor
// map over the array -- {128 four-bit elements, 128 rows, parts}, row pitch
// 64 B, part pitch PAD_MAT -- finds block b of row n at element 32 (b % 4) of
// row n % 128 in part (chunk_offset(n / 128, b / 4) + sub * PAD_MAT) / PAD_MAT,
// the part the kernel's producer asks for.  No two (n, b) share a byte.
static int check_padded(int N, int K, int NM) {
    for (int sub = 0; sub < NM; ++sub) {
        TiledMatrix M{nullptr, N, K, NM, sub, 1};
        const size_t total = M.expert_bytes();
        if (total != static_cast<size_t>(M.tiles()) * M.chunks() * NM * TiledMatrix::PAD_MAT)
            return fail("padded expert bytes", N, K, NM);
        std::vector<unsigned char> used(total, 0);
        for (int n = 0; n < N; ++n)
            for (int b = 0; b < M.nb(); ++b) {
                size_t co, so;
                M.locate(n, b, co, so);
                const int ft = n / 128, r = n % 128, c = b / 4, h = b % 4;
                const size_t off = M.chunk_offset(ft, c, 128) + static_cast<size_t>(sub) * TiledMatrix::PAD_MAT;
                if (off % TiledMatrix::PAD_MAT) return fail("part not aligned", N, n, b);
                const size_t part0 = off;   // part index * PAD_MAT
                if (co != part0 + static_cast<size_t>(r) * 64 + h * 16) return fail("padded code slot", N, n, b);
                if (so != part0 + 128 * 64 + 16 * (r % 32) + 4 * (r / 32) + h) return fail("padded scale byte", N, n, b);
                if (co + 16 > total || so >= total) return fail("padded slot outside the expert", N, n, b);
                for (int i = 0; i < 16; ++i)
                    if (used[co + i]++) return fail("padded code bytes shared", N, n, b);
                if (used[so]++) return fail("padded scale byte shared", N, n, b);
            }
    }
    return 0;
}

int main() {
    const int shapes[][3] = {{2880, 2880, 2}, {2880, 2880, 1}, {320, 192, 2}, {192, 320, 1},
                             {160, 96, 2},    {96, 160, 1},    {128, 64, 2},  {64, 128, 1}, {32, 32, 2}};
    for (auto& sh : shapes)
        if (check_matrix(sh[0], sh[1], sh[2]) || check_padded(sh[0], sh[1], sh[2])) return 1;
    std::vector<unsigned char> used(4 * 512, 0);
    for (int n = 0; n < 256; ++n)
        for (int q = 0; q < 4; ++q) {
            const unsigned o = sf_atom_offset(n, q);
            if (o >= 2 * 512) return fail("atom byte outside two atoms", n, q, static_cast<int>(o));
            if (o != static_cast<unsigned>((n / 128) * 512 + 16 * (n % 32) + 4 * ((n / 32) % 4) + q))
                return fail("atom byte formula", n, q, static_cast<int>(o));
            if (used[o]++) return fail("atom byte shared", n, q, static_cast<int>(o));
        }
    for (int i = 0; i < 2 * 512; ++i)
        if (!used[i]) return fail("atom byte unused", i, 0, 0);
    std::printf("ok\n");
    return 0;
}
