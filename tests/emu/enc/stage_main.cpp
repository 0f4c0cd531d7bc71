// Runs the two-launch encoder (code_buckets, then compact_stream), compiled for the
// host under block_emu.h, each grid with all its CTAs at once.
// argv: dir grid   (grid: CTAs of the bucket coder)
// dir holds params.bin (u64 n, d, s, seed, norm_kind, ef, cap_words) and in.bin
// (fp32[n]); with ef = 1 also e_in.bin (fp32[n]).  It writes words.bin
// (u32[cap_words]), offsets.bin (u64[nb + 1]), e_out.bin with ef = 1, and prints the
// status word.  The arguments and the workspace layout are those the library's host
// code derives.
#include "block_emu.h"
#include <cstdlib>
#include <algorithm>
thread_local dim3e threadIdx, blockIdx;
dim3e gridDim, blockDim;
thread_local BlockCtx* t_blk;
std::atomic<int> g_emu_error{0};
#include "stage_emu.inc"  // the kernel source, prepared by the test
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
static void code(const qsgd::StageArgs& a, unsigned grid, size_t smem) {
    if constexpr (kShort)
        run_grid(grid, qsgd::kStageBlock, smem, [&] { qsgd::code_buckets_short<V, kEF>(a); });
    else
        run_grid(grid, qsgd::kStageBlock, smem, [&] { qsgd::code_buckets<V, kEF>(a); });
}
template <int V, bool kEF>
static void code_v(const qsgd::StageArgs& a, unsigned grid, size_t smem) {
    if (a.s <= qsgd::kStageShortMaxS) code<V, true, kEF>(a, grid, smem); else code<V, false, kEF>(a, grid, smem);
}
template <bool kEF>
static void code_any(const qsgd::StageArgs& a, unsigned grid, size_t smem) {
    switch (qsgd::stage_v(a.d)) {
        case 1: code_v<1, kEF>(a, grid, smem); break;
        case 2: code_v<2, kEF>(a, grid, smem); break;
        case 4: code_v<4, kEF>(a, grid, smem); break;
        default: code_v<8, kEF>(a, grid, smem); break;
    }
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int main(int argc, char** argv) {
    const std::string dir = argv[1];
    const unsigned grid_req = std::atoi(argv[2]);
    auto prm = slurp(dir + "/params.bin");
    uint64_t q[7];
    std::memcpy(q, prm.data(), sizeof q);
    const uint64_t n = q[0], seed = q[3], cap = q[6];
    const uint32_t d = (uint32_t)q[1], s = (uint32_t)q[2], norm_kind = (uint32_t)q[4];
    const bool ef = q[5] != 0;
    auto inb = slurp(dir + "/in.bin");
    std::vector<float> in(n + 4), e(ef ? n + 4 : 0);  // 16-byte aligned by the allocator
    std::memcpy(in.data(), inb.data(), 4 * n);
    if (ef) {
        auto eb = slurp(dir + "/e_in.bin");
        std::memcpy(e.data(), eb.data(), 4 * n);
    }
    const uint64_t nb = (n + d - 1) / d;
    std::vector<uint32_t> words(cap, 0xDEADBEEFu);  // every word the stream covers is written
    std::vector<uint64_t> offsets(nb + 1, 0);
    uint32_t status = 0;
    // workspace as the host code lays it out: control block, descriptors, sizes, slots;
    // zeroed once, then filled with garbage where the kernels must not rely on zeros
    const uint64_t slot_bits = 32u + (uint64_t)d * (2u + qsgd::omega_len_host(s));
    // whole 16-byte units, as the library lays them out; STAGE_UNPADDED=1 lays them out
    // word by word, which the compaction must notice (it then copies without gathering)
    const bool unpadded = std::getenv("STAGE_UNPADDED") != nullptr;
    const uint32_t slot_words = unpadded ? (uint32_t)((slot_bits + 31) / 32) : (uint32_t)(((slot_bits + 31) / 32 + 3) / 4 * 4);
    const uint64_t ntiles = (nb + qsgd::kCompactBlock - 1) / qsgd::kCompactBlock;
    const size_t desc_off = 256, bits_off = desc_off + align256(8 * ntiles), stage_off = bits_off + align256(4 * nb);
    const size_t total = stage_off + align256(4 * nb * (size_t)slot_words);
    std::vector<uint64_t> ws((total + 7) / 8, 0);
    char* wsp = reinterpret_cast<char*>(ws.data());
    std::memset(wsp + desc_off, 0x5A, total - desc_off);  // an earlier call's leftovers
    qsgd::StageArgs a{};
    a.in = in.data();
    a.ef = ef ? e.data() : nullptr;
    a.n = n; a.d = d; a.s = s; a.norm_kind = norm_kind;
    const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    for (uint32_t r = 0; r < 10; ++r) {
        a.rk[2 * r] = k0 + r * 0x9E3779B9u;
        a.rk[2 * r + 1] = k1 + r * 0xBB67AE85u;
    }
    a.nb = nb;
    a.slot_words = slot_words;
    a.buf_words = slot_words + 1;
    a.stage = reinterpret_cast<uint32_t*>(wsp + stage_off);
    a.bits = reinterpret_cast<uint32_t*>(wsp + bits_off);
    a.status = &status;
    a.words = words.data(); a.cap_words = cap;
    a.offsets = offsets.data();
    a.ctrl = reinterpret_cast<qsgd::ScanControl*>(wsp);
    a.cdesc = reinterpret_cast<uint64_t*>(wsp + desc_off);
    a.ntiles = ntiles;
    const size_t smem = qsgd::stage_smem_bytes(s, a.buf_words);
    const unsigned grid = (unsigned)std::max<uint64_t>(1, std::min<uint64_t>((nb + qsgd::kStageWarps - 1) / qsgd::kStageWarps, grid_req));
    // two calls on the one workspace, the second over the first's leftovers; each call
    // must leave the control block at rest, and without memory the second call's
    // stream must equal the first's
    std::vector<uint32_t> first_words;
    std::vector<uint64_t> first_offsets;
    for (int call = 0; call < (ef ? 1 : 2); ++call) {
        if (ef) code_any<true>(a, grid, smem); else code_any<false>(a, grid, smem);
        if (g_emu_error) return 4;
        run_grid((unsigned)ntiles, qsgd::kCompactThreads, qsgd::kCompactSmemWords * 4, [&] { qsgd::compact_stream(a); });
        if (g_emu_error) return 4;
        const qsgd::ScanControl* c = reinterpret_cast<const qsgd::ScanControl*>(wsp);
        if (c->ticket != 0 || c->done != 0 || c->abort != 0) {
            std::fprintf(stderr, "control block not at rest after a call\n");
            return 5;
        }
        if (call == 0 && !ef) {
            first_words = words;
            first_offsets = offsets;
            std::fill(words.begin(), words.end(), 0xDEADBEEFu);
        } else if (call == 1 && (words != first_words || offsets != first_offsets)) {
            std::fprintf(stderr, "the second call's stream differs\n");
            return 6;
        }
    }
    spit(dir + "/words.bin", words.data(), 4 * cap);
    spit(dir + "/offsets.bin", offsets.data(), 8 * (nb + 1));
    if (ef) spit(dir + "/e_out.bin", e.data(), 4 * n);
    std::printf("status %u\n", status);
    return 0;
}
