// Runs the encoder kernels encode_fast and encode_general, compiled for the host
// under block_emu.h, with the whole grid at once.
// argv: dir mode grid   (mode 0: encode_fast, 1: encode_general)
// dir holds params.bin (u64 n, d, s, seed, norm_kind, ef, cap_words) and in.bin
// (fp32[n]); with ef = 1 also e_in.bin (fp32[n]).  It writes words.bin
// (u32[cap_words]), offsets.bin (u64[nb + 1]), e_out.bin with ef = 1, and prints the
// status word.  The arguments are those the library's host code derives.
#include "block_emu.h"
thread_local dim3e threadIdx, blockIdx;
dim3e gridDim, blockDim;
thread_local BlockCtx* t_blk;
std::atomic<int> g_emu_error{0};
#include "encode_emu.inc"  // the kernel source, prepared by the test
#include <string>

namespace qsgd {
uint32_t omega_len_host(uint64_t N) {
    uint32_t len = 1;
    while (N > 1) {
        uint32_t b = 0;
        for (uint64_t x = N; x; x >>= 1) ++b;
        len += b;
        N = b - 1;
    }
    return len;
}
}  // namespace qsgd

static std::vector<unsigned char> slurp(const std::string& p) {
    FILE* f = std::fopen(p.c_str(), "rb");
    if (!f) { std::perror(p.c_str()); std::exit(2); }
    std::fseek(f, 0, SEEK_END); long n = std::ftell(f); std::fseek(f, 0, SEEK_SET);
    std::vector<unsigned char> b(n);
    if (n && std::fread(b.data(), 1, n, f) != (size_t)n) std::exit(2);
    std::fclose(f);
    return b;
}
static void spit(const std::string& p, const void* data, size_t bytes) {
    FILE* f = std::fopen(p.c_str(), "wb");
    std::fwrite(data, 1, bytes, f);
    std::fclose(f);
}

template <class Kernel>
static void run_grid(unsigned grid, unsigned block, size_t smem, Kernel k) {
    gridDim = {grid, 1, 1};
    blockDim = {block, 1, 1};
    std::vector<std::unique_ptr<BlockCtx>> blocks;
    for (unsigned b = 0; b < grid; ++b) {
        blocks.emplace_back(new BlockCtx());
        blocks.back()->smem.assign(smem + 64, 0xAB);  // garbage, like real shared memory
    }
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

template <int V, bool kShort, bool kEF>
static void fast_kernel(const qsgd::EncodeArgs& a, unsigned grid, size_t smem) {
    run_grid(grid, qsgd::kFastBlock, smem, [&] { qsgd::encode_fast<V, kShort, kEF>(a); });
}
template <int V, bool kEF>
static void fast_v(const qsgd::EncodeArgs& a, unsigned grid, size_t smem) {
    if (a.s <= 31) fast_kernel<V, true, kEF>(a, grid, smem); else fast_kernel<V, false, kEF>(a, grid, smem);
}
template <bool kEF>
static void fast(const qsgd::EncodeArgs& a, unsigned grid, size_t smem) {
    switch (qsgd::fast_v(a.d)) {
        case 1: fast_v<1, kEF>(a, grid, smem); break;
        case 2: fast_v<2, kEF>(a, grid, smem); break;
        case 4: fast_v<4, kEF>(a, grid, smem); break;
        default: fast_v<8, kEF>(a, grid, smem); break;
    }
}

int main(int argc, char** argv) {
    const std::string dir = argv[1];
    const int mode = std::atoi(argv[2]);
    const unsigned grid_req = std::atoi(argv[3]);
    auto prm = slurp(dir + "/params.bin");
    uint64_t q[7];
    std::memcpy(q, prm.data(), sizeof q);
    const uint64_t n = q[0], seed = q[3], cap = q[6];
    const uint32_t d = (uint32_t)q[1], s = (uint32_t)q[2], norm_kind = (uint32_t)q[4];
    const bool ef = q[5] != 0;
    auto inb = slurp(dir + "/in.bin");
    std::vector<float> in(n), e(ef ? n : 0);
    std::memcpy(in.data(), inb.data(), 4 * n);
    if (ef) {
        auto eb = slurp(dir + "/e_in.bin");
        std::memcpy(e.data(), eb.data(), 4 * n);
    }
    const uint64_t nb = (n + d - 1) / d;
    std::vector<uint32_t> words(cap, 0xDEADBEEFu);  // every word the stream covers is written
    std::vector<uint64_t> offsets(nb + 1, 0);
    uint32_t status = 0;
    qsgd::EncodeArgs a{};
    a.in = in.data();
    a.n = n; a.d = d; a.s = s;
    a.key0 = (uint32_t)seed; a.key1 = (uint32_t)(seed >> 32);
    a.words = words.data(); a.cap_words = cap;
    a.offsets = offsets.data(); a.status = &status;
    a.norm_kind = norm_kind;
    a.ef = ef ? e.data() : nullptr;
    a.nb = nb;
    const uint32_t wl = 2u + qsgd::omega_len_host(s);
    size_t smem;
    unsigned block;
    if (mode == 0) {
        a.buckets_per_tile = qsgd::kFastWarps;
        a.ntiles = (nb + qsgd::kFastWarps - 1) / qsgd::kFastWarps;
        const uint64_t bits = (uint64_t)qsgd::kFastWarps * (32u + (uint64_t)d * wl);
        a.smem_words = (uint32_t)std::min<uint64_t>((bits + 31) / 32 + 2, 1u << 24);
        smem = qsgd::fast_smem_bytes(d, s, a.smem_words);
        block = qsgd::kFastBlock;
    } else {
        a.buckets_per_tile = d >= qsgd::kGeneralTileCoords ? 1u : qsgd::kGeneralTileCoords / d;
        a.ntiles = (nb + a.buckets_per_tile - 1) / a.buckets_per_tile;
        const uint64_t starts = qsgd::kChunk / d + 2;
        const uint64_t bits = 31u + (uint64_t)qsgd::kChunk * wl + 44u + qsgd::omega_len_host(s) + 32u * starts;
        a.smem_words = (uint32_t)((bits + 31) / 32 + 2);
        smem = qsgd::general_smem_bytes(a.smem_words, a.buckets_per_tile);
        block = qsgd::kBlock;
    }
    // workspace: control block, tile descriptors, tile states; zeroed once
    const size_t desc_off = 256;
    const size_t tiles_off = desc_off + ((sizeof(uint64_t) * ((a.ntiles + 1) & ~uint64_t(1)) + 255) & ~size_t(255));
    const size_t total = tiles_off + ((sizeof(qsgd::TileState) * a.ntiles + 255) & ~size_t(255));
    std::vector<uint64_t> ws((total + 7) / 8, 0);
    char* wsp = reinterpret_cast<char*>(ws.data());
    a.ctrl = reinterpret_cast<qsgd::ScanControl*>(wsp);
    a.tdesc = reinterpret_cast<uint64_t*>(wsp + desc_off);
    a.ts = reinterpret_cast<qsgd::TileState*>(wsp + tiles_off);
    const unsigned grid = (unsigned)std::max<uint64_t>(1, std::min<uint64_t>(a.ntiles, grid_req));
    if (mode == 0) {
        if (ef) fast<true>(a, grid, smem); else fast<false>(a, grid, smem);
    } else {
        run_grid(grid, block, smem, [&] { qsgd::encode_general(a); });
    }
    if (g_emu_error) return 4;
    spit(dir + "/words.bin", words.data(), 4 * cap);
    spit(dir + "/offsets.bin", offsets.data(), 8 * (nb + 1));
    if (ef) spit(dir + "/e_out.bin", e.data(), 4 * n);
    std::printf("status %u\n", status);
    return 0;
}
