// Runs the decoder kernels decode_multi (P = -1) and decode_warp (P = -2), compiled
// for the host under warp_emu.h, over streams read from files.
// argv: dir P accumulate [grid [mean]]
// dir holds params.bin (u64 n, d, s, K), out_in.bin (fp32[n]), w<j>.bin / o<j>.bin
// (words, offsets of stream j); the result goes to out.bin and the status to stdout.
// The K streams go 16 to a launch, as the library sends them; with mean = 1
// (decode_multi only) the first launch starts from +0 and the last divides by K.
#include "warp_emu.h"
thread_local dim3e threadIdx, blockIdx;
dim3e gridDim, blockDim;
unsigned char* g_emu_smem;
WarpSync* g_warps;
std::atomic<int> g_emu_error{0};
static std::mutex g_bm;
static std::condition_variable g_bcv;
static int g_barrived = 0;
static uint64_t g_bgen = 0;
void __syncthreads() {
    std::unique_lock<std::mutex> lk(g_bm);
    const uint64_t gen = g_bgen;
    if (++g_barrived == (int)blockDim.x) {
        g_barrived = 0;
        ++g_bgen;
        g_bcv.notify_all();
    } else if (!g_bcv.wait_for(lk, std::chrono::seconds(20), [&] { return g_bgen != gen; })) {
        emu_fail("__syncthreads timed out", 0);
        std::exit(3);
    }
}
#include "decode_emu.inc"  // the kernel source, prepared by the test
#include <string>
#include <thread>
static std::vector<unsigned char> slurp(const std::string& p) {
    FILE* f = std::fopen(p.c_str(), "rb");
    if (!f) { std::perror(p.c_str()); std::exit(2); }
    std::fseek(f, 0, SEEK_END); long n = std::ftell(f); std::fseek(f, 0, SEEK_SET);
    std::vector<unsigned char> b(n);
    if (n && std::fread(b.data(), 1, n, f) != (size_t)n) std::exit(2);
    std::fclose(f);
    return b;
}
template <bool A> static void run_warp(const qsgd::DecodeArgs& a, unsigned grid) {
    const int kBlock = qsgd::kDecodeBlock;
    const size_t smem = qsgd::kLut * 4 + (size_t)qsgd::kDecWarps * 32 * qsgd::kStride * 4 +
                        (size_t)kBlock * a.K * sizeof(qsgd::LaneStream);
    gridDim = {grid, 1, 1};
    blockDim = {(unsigned)kBlock, 1, 1};
    std::vector<unsigned char> sm(smem + 64);
    std::vector<WarpSync> warps(kBlock / 32);
    for (unsigned b = 0; b < grid; ++b) {
        g_emu_smem = sm.data();
        std::memset(sm.data(), 0xAB, sm.size());
        g_warps = warps.data();
        std::vector<std::thread> th;
        for (int t = 0; t < kBlock; ++t)
            th.emplace_back([&, t, b] {
                threadIdx = {(unsigned)t, 0, 0};
                blockIdx = {b, 0, 0};
                qsgd::decode_warp<A>(a);
            });
        for (auto& x : th) x.join();
    }
}

static void run_multi(const qsgd::DecodeArgs& a, unsigned grid) {
    const int kBlock = qsgd::kMultiBlock;
    const size_t smem = qsgd::kLut * 4 + (size_t)qsgd::kMultiWarps * 32 * qsgd::kMStride * 4;
    gridDim = {grid, 1, 1};
    blockDim = {(unsigned)kBlock, 1, 1};
    std::vector<unsigned char> sm(smem + 64);
    std::vector<WarpSync> warps(kBlock / 32);
    for (unsigned b = 0; b < grid; ++b) {
        g_emu_smem = sm.data();
        std::memset(sm.data(), 0xAB, sm.size());
        g_warps = warps.data();
        std::vector<std::thread> th;
        for (int t = 0; t < kBlock; ++t)
            th.emplace_back([&, t, b] {
                threadIdx = {(unsigned)t, 0, 0};
                blockIdx = {b, 0, 0};
                qsgd::decode_multi(a);
            });
        for (auto& x : th) x.join();
    }
}

int main(int argc, char** argv) {
    const std::string dir = argv[1];
    const int P = std::atoi(argv[2]);
    const bool acc = std::atoi(argv[3]) != 0;
    const unsigned grid = argc > 4 ? std::atoi(argv[4]) : 3;
    auto prm = slurp(dir + "/params.bin");  // u64 n, d, s, K
    uint64_t q[4];
    std::memcpy(q, prm.data(), 32);
    const uint64_t n = q[0];
    const uint32_t d = (uint32_t)q[1], s = (uint32_t)q[2];
    const int K = (int)q[3];
    auto outb = slurp(dir + "/out_in.bin");
    std::vector<float> out(n);
    std::memcpy(out.data(), outb.data(), 4 * n);
    uint32_t status = 0;
    std::vector<std::vector<unsigned char>> ws(K), os(K);
    if (P != -1 && P != -2) return 2;
    {
        const bool mean = argc > 5 && std::atoi(argv[5]) != 0;
        for (int j = 0; j < K; ++j) {
            ws[j] = slurp(dir + "/w" + std::to_string(j) + ".bin");
            os[j] = slurp(dir + "/o" + std::to_string(j) + ".bin");
        }
        for (int j0 = 0; j0 < K; j0 += qsgd::kMaxStreamsPerLaunch) {
            qsgd::DecodeArgs a{};
            a.n = n; a.d = d; a.s = s; a.nb = (n + d - 1) / d; a.out = out.data(); a.status = &status;
            a.K = std::min(K - j0, qsgd::kMaxStreamsPerLaunch);
            a.first_group = j0 == 0;
            a.start_zero = mean && j0 == 0;
            a.div = mean && j0 + a.K == K ? (float)K : 0.f;
            for (int j = 0; j < a.K; ++j) {
                a.streams[j].words = reinterpret_cast<const uint32_t*>(ws[j0 + j].data());
                a.streams[j].num_words = ws[j0 + j].size() / 4;
                a.streams[j].offsets = reinterpret_cast<const uint64_t*>(os[j0 + j].data());
            }
            if (P == -1)
                run_multi(a, grid);
            else if (acc)
                run_warp<true>(a, grid);
            else
                run_warp<false>(a, grid);
            if (g_emu_error) return 4;
        }
        FILE* f = std::fopen((dir + "/out.bin").c_str(), "wb");
        std::fwrite(out.data(), 4, n, f);
        std::fclose(f);
        std::printf("status %u\n", status);
        return 0;
    }
}
