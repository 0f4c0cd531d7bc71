// Runs the b-bit, error-feedback and mean kernels (qsgd_bbit.cu, qsgd_ef.cu,
// qsgd_mean.cu), compiled for the host under block_emu.h, on arrays read from files.
// argv: dir op grid.  params.bin holds u64 n, d, b_or_s, seed, norm_kind, flag, cap;
// the arrays a op reads and writes are named below.
#include "block_emu.h"
thread_local dim3e threadIdx, blockIdx;
dim3e gridDim, blockDim;
thread_local BlockCtx* t_blk;
std::atomic<int> g_emu_error{0};
#include "aux_emu.inc"  // the kernel sources, prepared by the test
#include <string>

template <class T> static std::vector<T> load(const std::string& p) {
    FILE* f = std::fopen(p.c_str(), "rb");
    if (!f) { std::perror(p.c_str()); std::exit(2); }
    std::fseek(f, 0, SEEK_END); long n = std::ftell(f); std::fseek(f, 0, SEEK_SET);
    std::vector<T> v(n / sizeof(T) + 1);
    if (n && std::fread(v.data(), 1, n, f) != (size_t)n) std::exit(2);
    std::fclose(f);
    return v;
}
template <class T> static void save(const std::string& p, const std::vector<T>& v, size_t count) {
    FILE* f = std::fopen(p.c_str(), "wb");
    std::fwrite(v.data(), sizeof(T), count, f);
    std::fclose(f);
}
template <class Kernel> static void run_grid(unsigned grid, unsigned block, Kernel k) {
    gridDim = {grid, 1, 1};
    blockDim = {block, 1, 1};
    std::vector<std::unique_ptr<BlockCtx>> blocks;
    for (unsigned b = 0; b < grid; ++b) blocks.emplace_back(new BlockCtx());
    std::vector<std::thread> th;
    for (unsigned b = 0; b < grid; ++b)
        for (unsigned t = 0; t < block; ++t)
            th.emplace_back([&, b, t] {
                t_blk = blocks[b].get();
                threadIdx = {t, 0, 0};
                blockIdx = {b, 0, 0};
                k();
            });
    for (auto& x : th) x.join();
}

using namespace qsgd;

template <int B, bool kEF>
static void bbit_fast(unsigned grid, const float* in, float* ef, uint64_t n, uint32_t d, uint64_t seed, uint32_t nk,
                      float* norms, uint32_t* codes, uint32_t* st) {
    switch (d / 128) {
        case 1: run_grid(grid, kBbitBlock, [&] { bbit_encode_fast<1, B, kEF>(in, ef, n, d, seed, nk, norms, codes, st); }); break;
        case 2: run_grid(grid, kBbitBlock, [&] { bbit_encode_fast<2, B, kEF>(in, ef, n, d, seed, nk, norms, codes, st); }); break;
        case 4: run_grid(grid, kBbitBlock, [&] { bbit_encode_fast<4, B, kEF>(in, ef, n, d, seed, nk, norms, codes, st); }); break;
        default: run_grid(grid, kBbitBlock, [&] { bbit_encode_fast<8, B, kEF>(in, ef, n, d, seed, nk, norms, codes, st); }); break;
    }
}
template <int B>
static void bbit_enc(unsigned grid, const float* in, float* ef, uint64_t n, uint32_t d, uint64_t seed, uint32_t nk,
                     float* norms, uint32_t* codes, uint32_t* st) {
    if (fast_shape(in, ef, d)) {
        if (ef) bbit_fast<B, true>(grid, in, ef, n, d, seed, nk, norms, codes, st);
        else bbit_fast<B, false>(grid, in, ef, n, d, seed, nk, norms, codes, st);
        return;
    }
    run_grid(grid, kBbitBlock, [&] { bbit_norms(in, n, d, (1u << (B - 1)) - 1u, nk, norms, st); });
    run_grid(grid, kBbitBlock, [&] { bbit_pack<B>(in, n, d, seed, norms, codes); });
}
template <int B>
static void bbit_dec(unsigned grid, bool vec, bool acc, const float* norms, const uint32_t* codes, uint64_t n,
                     uint32_t d, float* out, uint32_t* st) {
    if (vec) {
        if (acc) run_grid(grid, kBbitBlock, [&] { bbit_decode_vec<B, true>(norms, codes, n, d, out, st); });
        else run_grid(grid, kBbitBlock, [&] { bbit_decode_vec<B, false>(norms, codes, n, d, out, st); });
    } else {
        if (acc) run_grid(grid, kBbitBlock, [&] { bbit_decode_scalar<B, true>(norms, codes, n, d, out, st); });
        else run_grid(grid, kBbitBlock, [&] { bbit_decode_scalar<B, false>(norms, codes, n, d, out, st); });
    }
}

int main(int argc, char** argv) {
    const std::string dir = argv[1], op = argv[2];
    const unsigned grid = std::atoi(argv[3]);
    auto q = load<uint64_t>(dir + "/params.bin");
    const uint64_t n = q[0], seed = q[3], cap = q[6];
    const uint32_t d = (uint32_t)q[1], bs = (uint32_t)q[2], nk = (uint32_t)q[4], flag = (uint32_t)q[5];
    const uint64_t nb = (n + d - 1) / d;
    uint32_t st = 0;
    if (op == "bbit_enc") {  // in.bin [+ e.bin when flag]; writes norms.bin, codes.bin [, e_out.bin]
        auto in = load<float>(dir + "/in.bin");
        std::vector<float> e = flag ? load<float>(dir + "/e.bin") : std::vector<float>();
        std::vector<float> norms(nb + 1, 0.f);
        const uint64_t cw = (n * bs + 31) / 32;
        std::vector<uint32_t> codes(cw + 1, 0xDEADBEEFu);
        float* ef = flag ? e.data() : nullptr;
        if (bs == 2) bbit_enc<2>(grid, in.data(), ef, n, d, seed, nk, norms.data(), codes.data(), &st);
        else if (bs == 4) bbit_enc<4>(grid, in.data(), ef, n, d, seed, nk, norms.data(), codes.data(), &st);
        else bbit_enc<8>(grid, in.data(), ef, n, d, seed, nk, norms.data(), codes.data(), &st);
        save(dir + "/norms.bin", norms, nb);
        save(dir + "/codes.bin", codes, cw);
        if (flag) save(dir + "/e_out.bin", e, n);
    } else if (op == "bbit_dec" || op == "bbit_acc") {  // norms.bin, codes.bin, out.bin; flag: vector form
        auto norms = load<float>(dir + "/norms.bin");
        auto codes = load<uint32_t>(dir + "/codes.bin");
        auto out = load<float>(dir + "/out.bin");
        const bool acc = op == "bbit_acc";
        if (bs == 2) bbit_dec<2>(grid, flag != 0, acc, norms.data(), codes.data(), n, d, out.data(), &st);
        else if (bs == 4) bbit_dec<4>(grid, flag != 0, acc, norms.data(), codes.data(), n, d, out.data(), &st);
        else bbit_dec<8>(grid, flag != 0, acc, norms.data(), codes.data(), n, d, out.data(), &st);
        save(dir + "/out.bin", out, n);
    } else if (op == "ef_add") {  // g.bin, e.bin -> e.bin; flag: vector form
        auto g = load<float>(dir + "/g.bin");
        auto e = load<float>(dir + "/e.bin");
        if (flag) run_grid(grid, kEfBlock, [&] { ef_add<true>(g.data(), e.data(), n); });
        else run_grid(grid, kEfBlock, [&] { ef_add<false>(g.data(), e.data(), n); });
        save(dir + "/e.bin", e, n);
    } else if (op == "ef_res_elias") {  // e.bin (holding p), words.bin, offsets.bin -> e.bin
        auto e = load<float>(dir + "/e.bin");
        auto words = load<uint32_t>(dir + "/words.bin");
        auto offsets = load<uint64_t>(dir + "/offsets.bin");
        const PhiloxKey key{(uint32_t)seed, (uint32_t)(seed >> 32)};
        run_grid(grid, kEfBlock, [&] { ef_residual_elias(e.data(), words.data(), cap, offsets.data(), n, d, bs, key); });
        save(dir + "/e.bin", e, n);
    } else if (op == "ef_res_bbit") {  // e.bin (holding p), norms.bin, codes.bin -> e.bin
        auto e = load<float>(dir + "/e.bin");
        auto norms = load<float>(dir + "/norms.bin");
        auto codes = load<uint32_t>(dir + "/codes.bin");
        if (bs == 2) run_grid(grid, kEfBlock, [&] { ef_residual_bbit<2>(e.data(), norms.data(), codes.data(), n, d); });
        else if (bs == 4) run_grid(grid, kEfBlock, [&] { ef_residual_bbit<4>(e.data(), norms.data(), codes.data(), n, d); });
        else run_grid(grid, kEfBlock, [&] { ef_residual_bbit<8>(e.data(), norms.data(), codes.data(), n, d); });
        save(dir + "/e.bin", e, n);
    } else if (op == "div") {  // out.bin -> out.bin divided by bs; flag: vector form
        auto out = load<float>(dir + "/out.bin");
        const float k = (float)bs;
        if (flag) run_grid(grid, kDivBlock, [&] { div_by<true>(out.data(), n, k); });
        else run_grid(grid, kDivBlock, [&] { div_by<false>(out.data(), n, k); });
        save(dir + "/out.bin", out, n);
    } else {
        std::fprintf(stderr, "unknown op %s\n", op.c_str());
        return 2;
    }
    if (g_emu_error) return 4;
    std::printf("status %u\n", st);
    return 0;
}
