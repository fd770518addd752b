// plan_check.cu -- host-only checks of the kernels' launch plans and work splits.
//
// Built by tests/test_plan_check.py with nvcc and run on the CPU: it calls only the
// __host__ functions of the kernel headers (plans, unit ranges, the fix-up rule) and
// makes no CUDA call, so it needs no GPU.  Each check compares the product's rule with
// ground truth computed here from the unit intervals themselves.  Prints one line per
// failure and "plan_check ok <checks>" at the end; the exit status is the failure count
// (capped at 100).
#include <cstdio>
#include <cstdlib>
#include <map>
#include <set>
#include <vector>

#include "../w3a16_gemv_b200/csrc/decode_split.cuh"
#include "../w3a16_gemv_b200/csrc/decode_streamk.cuh"
#define W3_TC_NS decode_tc32
#define W3_TC_BATCH 32
#include "../w3a16_gemv_b200/csrc/decode_tcgen05.cuh"
#include "../w3a16_gemv_b200/csrc/prefill_gemm.cuh"
#include "../w3a16_gemv_b200/csrc/prefill_swab.cuh"

namespace {

long g_checks = 0, g_fail = 0;

#define CHECK(cond, ...)                                   \
    do {                                                   \
        ++g_checks;                                        \
        if (!(cond)) {                                     \
            ++g_fail;                                      \
            if (g_fail <= 40) {                            \
                std::printf("FAIL %s:%d ", __FILE__, __LINE__); \
                std::printf(__VA_ARGS__);                  \
                std::printf("\n");                         \
            }                                              \
        }                                                  \
    } while (0)

const int kSmsList[] = {1, 2, 7, 100, 132, 148, 160};
const int kNList[] = {32, 40, 255, 256, 257, 300, 512, 1000, 1024, 4096, 4800, 8192, 10240, 28416, 28672, 57344};
const int kKList[] = {128, 256, 384, 1024, 1152, 4096, 8192, 28672};

// ---- 32-wide tensor-core decode: stream-K ranges over (256-row tile, group) units, shared
//      tiles finished by the fix-up kernel ----
void check_tc32(int N, int K, int sms) {
    namespace T = w3::decode_tc32;
    const T::LaunchPlan L = T::plan(N, K, sms);
    const int G = K / 128;
    const int64_t tiles = (N + T::kRows - 1) / T::kRows;
    const int64_t U = tiles * G;
    const int P = L.P;
    CHECK(L.U == U, "tc32 N=%d K=%d sms=%d: U %lld != %lld", N, K, sms, (long long)L.U, (long long)U);
    CHECK(P >= 1 && P <= sms * T::kCtasPerSm, "tc32 N=%d K=%d sms=%d: P=%d", N, K, sms, P);
    CHECK(L.ws_floats == (P > 1 ? int64_t(P) * 2 * T::kBatch * T::kRows : 0), "tc32 workspace N=%d K=%d", N, K);
    // each tile: CTAs whose range meets it (ground truth from the intervals), direct writers,
    // and the (CTA, slot) pairs that hold its partial sums
    std::vector<std::vector<int>> holders(tiles);
    std::vector<int> direct(tiles, 0);
    std::vector<std::map<int, int>> parts(tiles);
    for (int c = 0; c < P; ++c) {
        const int64_t b0 = T::unit_begin(c, U, P), b1 = T::unit_begin(c + 1, U, P);
        CHECK(b1 > b0, "tc32 N=%d K=%d sms=%d: CTA %d has no units", N, K, sms, c);
        for (int64_t t = b0 / G; t < tiles && t * G < b1; ++t) holders[t].push_back(c);
        T::Walk w(c, U, P, G);
        int64_t t, covered = 0, prev_end = b0;
        int g0, len;
        std::set<int> slots_used;
        while (w.next(t, g0, len)) {
            CHECK(t * G + g0 == prev_end && len >= 1 && g0 + len <= G, "tc32 walk N=%d K=%d CTA %d", N, K, c);
            prev_end = t * G + g0 + len;
            covered += len;
            if (len == G) {
                ++direct[t];
            } else {
                const int s = T::partial_slot(c, t, U, P, G);
                CHECK(s == 0 || s == 1, "tc32 slot");
                CHECK(slots_used.insert(s).second, "tc32 N=%d K=%d CTA %d: two shared tiles in slot %d", N, K, c, s);
                parts[t][c] = s;
            }
        }
        CHECK(covered == b1 - b0, "tc32 N=%d K=%d CTA %d: walk covers %lld of %lld units", N, K, c,
              (long long)covered, (long long)(b1 - b0));
    }
    std::vector<int> finisher(tiles, -1);
    for (int b = 0; b + 1 < P; ++b) {
        const int64_t t = T::fixup_tile(b, U, P, G);
        if (t < 0) continue;
        CHECK(t < tiles && finisher[t] < 0, "tc32 N=%d K=%d: tile %lld finished twice", N, K, (long long)t);
        if (t >= tiles) continue;
        finisher[t] = b;
        std::vector<int> contrib;
        for (int c = b; T::holds_part(c, t, U, P, G); ++c) {
            contrib.push_back(c);
            const auto it = parts[t].find(c);
            CHECK(it != parts[t].end() && it->second == T::partial_slot(c, t, U, P, G),
                  "tc32 N=%d K=%d: fix-up of tile %lld reads CTA %d slot %d, not written", N, K, (long long)t, c,
                  T::partial_slot(c, t, U, P, G));
        }
        CHECK(contrib == holders[t], "tc32 N=%d K=%d sms=%d: tile %lld contributors differ", N, K, sms, (long long)t);
    }
    for (int64_t t = 0; t < tiles; ++t) {
        if (holders[t].size() == 1) {
            CHECK(direct[t] == 1 && finisher[t] < 0 && parts[t].empty(), "tc32 N=%d K=%d: whole tile %lld", N, K,
                  (long long)t);
        } else {
            CHECK(direct[t] == 0 && finisher[t] >= 0 && parts[t].size() == holders[t].size(),
                  "tc32 N=%d K=%d sms=%d: shared tile %lld (holders %zu, finisher %d, parts %zu)", N, K, sms,
                  (long long)t, holders[t].size(), finisher[t], parts[t].size());
        }
    }
}

// ---- split decode: clusters own block ranges, ranks own K slices, warps stream-K ranges ----
void check_split(int M, int N, int K, int sms, int occupancy_mode) {
    namespace D = w3::dsplit;
    auto active = [&](int C, int smem) -> int {
        (void)smem;
        if (occupancy_mode == 0) return 0;           // the device cannot say
        if (occupancy_mode == 1) return sms / C;     // every SM holds one CTA
        return (sms / C) / 2 > 0 ? (sms / C) / 2 : 1;  // fewer clusters fit than SMs / C
    };
    const D::LaunchPlan L = D::plan(M, N, K, sms, active);
    const int G = K / 128;
    const int NB = (N + D::kBlockRows - 1) / D::kBlockRows;
    // Whether a plan exists must not depend on the occupancy answer: the route query (which
    // touches no device) asks with "cannot say", the launch with the device's answer.
    const bool ok_unknown = D::plan(M, N, K, sms, [](int, int) { return 0; }).ok;
    CHECK(L.ok == ok_unknown, "split M=%d N=%d K=%d sms=%d: plan exists %d with the occupancy answer, %d without",
          M, N, K, sms, int(L.ok), int(ok_unknown));
    if (!L.ok) return;
    CHECK(L.mt >= M && (L.mt == 1 || L.mt == 2 || L.mt == 4 || L.mt == 8 || L.mt == 16), "split mt=%d M=%d", L.mt, M);
    CHECK((L.C == 1 || L.C == 2 || L.C == 4 || L.C == 8) && L.C <= G, "split C=%d G=%d", L.C, G);
    CHECK(L.ncl >= 1 && L.ncl <= NB && int64_t(L.ncl) * L.C <= sms, "split M=%d N=%d K=%d sms=%d: %d clusters of %d",
          M, N, K, sms, L.ncl, L.C);
    // more clusters than are resident at once only when the resident ones' larger share of
    // blocks would not fit in shared memory (the clusters then run in waves)
    if (occupancy_mode == 2 && L.C > 1) {
        const int fit = active(L.C, 0);
        CHECK(L.ncl <= fit || D::fitting_depth(L.gs_max, L.mt, (NB + fit - 1) / fit, L.C) == 0,
              "split M=%d N=%d K=%d sms=%d: %d clusters, %d resident", M, N, K, sms, L.ncl, fit);
    }
    CHECK(L.depth >= 2 && L.depth <= D::kMaxDepth, "split depth %d", L.depth);
    CHECK(L.smem_bytes == D::smem_layout(L.gs_max, L.mt, L.depth, L.nb_max, L.C).total &&
              L.smem_bytes <= D::kSmemLimit,
          "split M=%d N=%d K=%d: shared memory %d", M, N, K, L.smem_bytes);
    // the cluster block ranges and the rank slices tile the matrix; every CTA's share fits the
    // shared memory sized by (gs_max, nb_max); the warps' unit ranges tile each CTA's units
    int64_t blocks = 0;
    for (int cl = 0; cl < L.ncl; ++cl) {
        const int b0 = int(int64_t(NB) * cl / L.ncl), b1 = int(int64_t(NB) * (cl + 1) / L.ncl);
        CHECK(b1 - b0 <= L.nb_max, "split: cluster %d has %d blocks > %d", cl, b1 - b0, L.nb_max);
        blocks += b1 - b0;
        int gsum = 0;
        for (int q = 0; q < L.C; ++q) {
            const int g0 = G * q / L.C, gs = G * (q + 1) / L.C - g0;
            CHECK(g0 == gsum && gs >= 1 && gs <= L.gs_max, "split: rank %d slice [%d, +%d)", q, g0, gs);
            gsum += gs;
            const int64_t units = int64_t(b1 - b0) * gs;
            int64_t prev = 0;
            for (int w = 0; w < D::kWarps; ++w) {
                int64_t u0, u1;
                D::warp_range(units, w, D::kWarps, u0, u1);
                CHECK(u0 == prev && u1 >= u0, "split: warp %d range", w);
                prev = u1;
            }
            CHECK(prev == units, "split: warps cover %lld of %lld units", (long long)prev, (long long)units);
        }
        CHECK(gsum == G, "split: slices cover %d of %d groups", gsum, G);
    }
    CHECK(blocks == NB, "split M=%d N=%d: clusters cover %lld of %d blocks", M, N, (long long)blocks, NB);
}

// ---- stream-K decode (M <= 4) ----
void check_sk(int M, int N, int K, int sms) {
    namespace S = w3::decode_sk;
    if (!S::applicable(M, N, K)) return;
    const S::LaunchPlan L = S::plan(M, N, K, sms);
    const int NB = (N + S::kBlockRows - 1) / S::kBlockRows;
    CHECK(L.ctas >= 1 && L.ctas <= sms && L.ctas <= NB, "sk M=%d N=%d K=%d sms=%d: %d CTAs", M, N, K, sms, L.ctas);
    CHECK(L.depth >= 2 && L.smem_bytes <= S::kSmemLimit, "sk M=%d N=%d K=%d: depth %d smem %d", M, N, K, L.depth,
          L.smem_bytes);
    CHECK(L.mt >= M && L.mt <= 4, "sk mt");
}

// ---- the two prefill kernels: their grids cover every (x row, W row) once ----
void check_prefill(int M, int N, int sms) {
    namespace F = w3::prefill;
    namespace A = w3::prefill_ab;
    const F::LaunchPlan P = F::plan(M, N, sms);
    const int mt = (M + F::kTileM - 1) / F::kTileM;
    CHECK(P.tile_n % 32 == 0 && P.tile_n >= 32 && P.tile_n <= F::kMaxTileN && (N < 128 || P.tile_n >= 128),
          "prefill M=%d N=%d: tile_n %d", M, N, P.tile_n);
    const int64_t ntiles = (N + P.tile_n - 1) / P.tile_n;
    CHECK(int64_t(P.grid.x) == mt * ntiles && int64_t(P.tile_n) * ntiles >= N && int64_t(P.tile_n) * (ntiles - 1) < N,
          "prefill M=%d N=%d: grid %u", M, N, P.grid.x);
    const A::LaunchPlan Q = A::plan(M, N);
    CHECK(Q.bn % 16 == 0 && Q.bn >= 16 && Q.bn <= A::kMaxBN && int64_t(Q.bn) * Q.xtiles >= M &&
              int64_t(Q.bn) * (Q.xtiles - 1) < M,
          "prefill_ab M=%d: bn %d x %d", M, Q.bn, Q.xtiles);
    CHECK(int64_t(Q.grid.x) == int64_t(Q.xtiles) * ((N + A::kRowsW - 1) / A::kRowsW), "prefill_ab M=%d N=%d grid", M,
          N);
}

}  // namespace

int main() {
    for (int sms : kSmsList)
        for (int N : kNList)
            for (int K : kKList) {
                if (N >= 256) check_tc32(N, K, sms);
                for (int M : {5, 8, 9, 12, 16}) {
                    if (M != 16 && M != 5 && sms != 148) continue;
                    for (int mode = 0; mode < 3; ++mode) check_split(M, N, K, sms, mode);
                }
                for (int M = 1; M <= 4; ++M) check_sk(M, N, K, sms);
            }
    // a stride of odd sizes for the tile arithmetic of the fix-up
    for (int N = 256; N <= 20000; N += 997)
        for (int K = 128; K <= 4096; K += 640)
            for (int sms : {148, 37}) check_tc32(N, K, sms);
    for (int sms : {1, 148})
        for (int N : kNList)
            for (int M : {17, 33, 64, 100, 128, 129, 200, 255, 256, 257, 300, 513, 1024, 2048, 4096}) check_prefill(M, N, sms);
    std::printf("plan_check ok %ld checks, %ld failures\n", g_checks, g_fail);
    return g_fail > 100 ? 100 : static_cast<int>(g_fail);
}
