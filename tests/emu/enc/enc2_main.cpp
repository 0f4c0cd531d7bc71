// Runs the two-pass encoder (qsgd_encode2.cu: levels, scan, pack) under block_emu.h.
// argv: dir grid
// params.bin: u64 n, d, s, seed, norm_kind, cap_words; in.bin fp32[n].
#include "block_emu.h"
thread_local dim3e threadIdx, blockIdx;
dim3e gridDim, blockDim;
thread_local BlockCtx* t_blk;
std::atomic<int> g_emu_error{0};
#include "encode2_emu.inc"  // the kernel source, prepared by the test
#include <string>
namespace qsgd {
uint32_t omega_len_host(uint64_t N) {
    uint32_t len = 1;
    while (N > 1) { uint32_t b = 0; for (uint64_t x = N; x; x >>= 1) ++b; len += b; N = b - 1; }
    return len;
}
}
template <class T> static std::vector<T> load(const std::string& p) {
    FILE* f = std::fopen(p.c_str(), "rb"); if (!f) std::exit(2);
    std::fseek(f, 0, SEEK_END); long n = std::ftell(f); std::fseek(f, 0, SEEK_SET);
    std::vector<T> v(n / sizeof(T) + 1); if (n && std::fread(v.data(), 1, n, f) != (size_t)n) std::exit(2); std::fclose(f); return v;
}
template <class T> static void save(const std::string& p, const T* v, size_t count) {
    FILE* f = std::fopen(p.c_str(), "wb"); std::fwrite(v, sizeof(T), count, f); std::fclose(f);
}
template <class Kernel> static void run_grid(unsigned grid, unsigned block, size_t smem, Kernel k) {
    gridDim = {grid, 1, 1}; blockDim = {block, 1, 1};
    std::vector<std::unique_ptr<BlockCtx>> blocks;
    for (unsigned b = 0; b < grid; ++b) { blocks.emplace_back(new BlockCtx()); blocks.back()->smem.assign(smem + 64, 0xAB); }
    std::vector<std::thread> th;
    for (unsigned b = 0; b < grid; ++b)
        for (unsigned t = 0; t < block; ++t)
            th.emplace_back([&, b, t] { t_blk = blocks[b].get(); threadIdx = {t, 0, 0}; blockIdx = {b, 0, 0}; k(); });
    for (auto& x : th) x.join();
}
using namespace qsgd;
template <int V> static void passes(const Enc2Args& a, unsigned grid) {
    run_grid(grid, kE2Block, ((size_t)kOmegaTab + (size_t)kE2Warps * 128 * V) * 4, [&] { enc2_levels<V>(a); });
    run_grid(1, kScanBlock, 0, [&] { enc2_scan(a); });
    const bool sh = a.s <= 31;
    const size_t smem = (kRecordTab + (size_t)kE2Warps * a.bucket_words + (size_t)kE2Warps * 32 * fast_lane_words(V, sh)) * 4;
    if (sh) run_grid(grid, kE2Block, smem, [&] { enc2_pack<V, true>(a); });
    else run_grid(grid, kE2Block, smem, [&] { enc2_pack<V, false>(a); });
}
int main(int argc, char** argv) {
    const std::string dir = argv[1];
    const unsigned grid = std::atoi(argv[2]);
    auto q = load<uint64_t>(dir + "/params.bin");
    const uint64_t n = q[0], seed = q[3], cap = q[5];
    const uint32_t d = (uint32_t)q[1], s = (uint32_t)q[2], nk = (uint32_t)q[4];
    auto in = load<float>(dir + "/in.bin");
    const uint64_t nb = (n + d - 1) / d;
    std::vector<uint32_t> recs(nb * d + 1), nz(nb + 1), bits(nb + 1), words(cap + 1, 0xDEADBEEFu);
    std::vector<float> norms(nb + 1);
    std::vector<uint64_t> offsets(nb + 1);
    uint32_t status = 0;
    Enc2Args a{};
    a.in = in.data(); a.n = n; a.d = d; a.s = s; a.key0 = (uint32_t)seed; a.key1 = (uint32_t)(seed >> 32); a.norm_kind = nk;
    a.nb = nb; a.recs = recs.data(); a.nz = nz.data(); a.bits = bits.data(); a.norms = norms.data();
    a.offsets = offsets.data(); a.words = words.data(); a.cap_words = cap; a.status = &status;
    a.bucket_words = (uint32_t)std::max<uint64_t>((32u + (uint64_t)d * (2u + omega_len_host(s)) + 31) / 32 + 1, d);
    switch (fast_v(d)) {
        case 1: passes<1>(a, grid); break;
        case 2: passes<2>(a, grid); break;
        case 4: passes<4>(a, grid); break;
        default: passes<8>(a, grid); break;
    }
    if (g_emu_error) return 4;
    save(dir + "/words.bin", words.data(), cap);
    save(dir + "/offsets.bin", offsets.data(), nb + 1);
    std::printf("status %u\n", status);
    return 0;
}
