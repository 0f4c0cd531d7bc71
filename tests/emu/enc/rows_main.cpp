// Runs the row decoders (decode_rows, decode_rows_ring, decode_rows_multi,
// decode_rows_side, and for large buckets sparse_fill with sparse_records or
// decode_sparse_acc), compiled for the host under block_emu.h, with all
// their CTAs at once.
// argv: dir accumulate grid warps [K [mean [side]]]
// dir holds params.bin (u64 n, d, s), w<j>.bin (u32 stream words), o<j>.bin
// (u64[nb+1]) and out_in.bin (fp32[n], the output before the call).  It writes
// out.bin and prints the status word.
#include "block_emu.h"
thread_local dim3e threadIdx, blockIdx;
dim3e gridDim, blockDim;
thread_local BlockCtx* t_blk;
std::atomic<int> g_emu_error{0};
#include "rows_emu.inc"  // the kernel source, prepared by the test
#include <string>

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

template <int V>
static void run_v(const qsgd::DecodeArgs& a, bool acc, unsigned grid, unsigned W, uint32_t stride, size_t smem) {
    if (acc)
        run_grid(grid, 32 * W, smem, [&] { qsgd::decode_rows<V, true>(a, stride); });
    else
        run_grid(grid, 32 * W, smem, [&] { qsgd::decode_rows<V, false>(a, stride); });
}
template <class T>
static void run_t(const qsgd::DecodeArgs& a, bool acc, unsigned grid, unsigned W) {
    if constexpr (sizeof(T) == 2) {
        const uint32_t stride = qsgd::ring_stride_words();
        const size_t smem = 4 * (size_t)(qsgd::kLutSize + qsgd::kSmallLutWords) + (size_t)W * 32 * stride * 4 +
                            (size_t)W * 32 * 8 * 4;
        if (acc)
            run_grid(grid, 32 * W, smem, [&] { qsgd::decode_rows_ring<true>(a, stride); });
        else
            run_grid(grid, 32 * W, smem, [&] { qsgd::decode_rows_ring<false>(a, stride); });
        return;
    }
    const uint32_t stride = qsgd::rows_stride_words(a.d);
    const size_t smem = 4 * (size_t)(qsgd::kLutSize + qsgd::kSmallLutWords) + (size_t)W * 32 * stride * 4;
    switch (qsgd::fast_v(a.d)) {
        case 1: run_v<1>(a, acc, grid, W, stride, smem); break;
        case 2: run_v<2>(a, acc, grid, W, stride, smem); break;
        case 4: run_v<4>(a, acc, grid, W, stride, smem); break;
        default: run_v<8>(a, acc, grid, W, stride, smem); break;
    }
}

// Several streams: decode_rows_multi over K streams, 16 to a launch as the library
// sends them (a mean starts the first launch from +0 and divides in the last); with
// side, decode_rows_side (a CTA of kSideWarps warps, the streams side by side).
static void run_multi(qsgd::DecodeArgs a, const std::vector<std::vector<unsigned char>>& ws,
                      const std::vector<std::vector<unsigned char>>& os, bool mean, unsigned grid, unsigned W,
                      bool side) {
    const int K = (int)ws.size();
    const size_t smem = side ? (qsgd::kLutSize + qsgd::kSmallLutWords + 32 * qsgd::kSideWarps +
                                (size_t)32 * qsgd::kSideWarps * qsgd::kSStride) * 4
                             : (qsgd::kLutSize + 256) * 2 + (size_t)W * (sizeof(qsgd::MsState) + 32 * qsgd::kMTile * 4);
    for (int j0 = 0; j0 < K; j0 += qsgd::kMaxStreamsPerLaunch) {
        a.K = std::min(K - j0, qsgd::kMaxStreamsPerLaunch);
        a.first_group = j0 == 0;
        a.start_zero = mean && j0 == 0;
        a.div = mean && j0 + a.K == K ? (float)K : 0.f;
        for (int j = 0; j < a.K; ++j) {
            a.streams[j].words = reinterpret_cast<const uint32_t*>(ws[j0 + j].data());
            a.streams[j].num_words = ws[j0 + j].size() / 4;
            a.streams[j].offsets = reinterpret_cast<const uint64_t*>(os[j0 + j].data());
        }
        if (side)
            run_grid(grid, 32 * qsgd::kSideWarps, smem, [&] { qsgd::decode_rows_side(a); });
        else
            run_grid(grid, 32 * W, smem, [&] { qsgd::decode_rows_multi(a); });
        if (g_emu_error) return;
    }
}

int main(int argc, char** argv) {
    const std::string dir = argv[1];
    const bool acc = std::atoi(argv[2]) != 0;
    const unsigned grid = std::atoi(argv[3]), W = std::atoi(argv[4]);
    const int K = argc > 5 ? std::atoi(argv[5]) : 1;
    const bool mean = argc > 6 && std::atoi(argv[6]) != 0;
    const bool side = argc > 7 && std::atoi(argv[7]) != 0;
    auto prm = slurp(dir + "/params.bin");
    uint64_t q[3];
    std::memcpy(q, prm.data(), sizeof q);
    const uint64_t n = q[0];
    const uint32_t d = (uint32_t)q[1], s = (uint32_t)q[2];
    const uint64_t nb = (n + d - 1) / d;
    auto wb = slurp(dir + "/w0.bin");
    auto ob = slurp(dir + "/o0.bin");
    auto xb = slurp(dir + "/out_in.bin");
    std::vector<uint32_t> words(wb.size() / 4 + 1);
    std::memcpy(words.data(), wb.data(), wb.size());
    std::vector<uint64_t> offsets(nb + 1);
    std::memcpy(offsets.data(), ob.data(), 8 * (nb + 1));
    std::vector<float> out(n + 4);
    std::memcpy(out.data(), xb.data(), 4 * n);
    uint32_t status = 0;
    if (d > qsgd::kRowsMaxD) {  // the large-bucket decoder, 16 streams to a launch
        std::vector<std::vector<unsigned char>> ws(K), os(K);
        for (int j = 0; j < K; ++j) {
            ws[j] = slurp(dir + "/w" + std::to_string(j) + ".bin");
            os[j] = slurp(dir + "/o" + std::to_string(j) + ".bin");
        }
        for (int j0 = 0; j0 < K; j0 += qsgd::kMaxStreamsPerLaunch) {
            qsgd::DecodeArgs a{};
            a.n = n; a.d = d; a.s = s; a.nb = nb; a.out = out.data(); a.status = &status;
            a.K = std::min(K - j0, qsgd::kMaxStreamsPerLaunch);
            a.first_group = j0 == 0;
            for (int j = 0; j < a.K; ++j) {
                a.streams[j].words = reinterpret_cast<const uint32_t*>(ws[j0 + j].data());
                a.streams[j].num_words = ws[j0 + j].size() / 4;
                a.streams[j].offsets = reinterpret_cast<const uint64_t*>(os[j0 + j].data());
            }
            if (acc) {
                run_grid(grid, qsgd::kSparseBlock, 0, [&] { qsgd::decode_sparse_acc(a); });
            } else {  // the fill (grid CTAs, grid-stride), then a lane a bucket
                run_grid(grid, qsgd::kSparseBlock, 0, [&] { qsgd::sparse_fill(a.out, a.n); });
                if (g_emu_error) return 4;
                run_grid((unsigned)((nb + qsgd::kSparseRecBuckets - 1) / qsgd::kSparseRecBuckets), qsgd::kSparseRecBlock, 0,
                         [&] { qsgd::sparse_records(a); });
            }
            if (g_emu_error) return 4;
        }
        spit(dir + "/out.bin", out.data(), 4 * n);
        std::printf("status %u\n", status);
        return 0;
    }
    if (K > 1 || mean) {
        std::vector<std::vector<unsigned char>> ws(K), os(K);
        for (int j = 0; j < K; ++j) {
            ws[j] = slurp(dir + "/w" + std::to_string(j) + ".bin");
            os[j] = slurp(dir + "/o" + std::to_string(j) + ".bin");
        }
        qsgd::DecodeArgs a{};
        a.n = n; a.d = d; a.s = s; a.nb = nb; a.out = out.data(); a.status = &status;
        run_multi(a, ws, os, mean, grid, W, side);
        if (g_emu_error) return 4;
        spit(dir + "/out.bin", out.data(), 4 * n);
        std::printf("status %u\n", status);
        return 0;
    }
    qsgd::DecodeArgs a{};
    a.streams[0].words = words.data();
    a.streams[0].num_words = wb.size() / 4;
    a.streams[0].offsets = offsets.data();
    a.K = 1;
    a.n = n; a.d = d; a.s = s; a.nb = nb;
    a.out = out.data();
    a.status = &status;
    a.first_group = 1;
    if (s <= qsgd::kRowsMaxS8)
        run_t<uint8_t>(a, acc, grid, W);
    else
        run_t<uint16_t>(a, acc, grid, W);
    if (g_emu_error) return 4;
    spit(dir + "/out.bin", out.data(), 4 * n);
    std::printf("status %u\n", status);
    return 0;
}
