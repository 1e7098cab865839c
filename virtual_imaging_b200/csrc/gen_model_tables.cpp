// gen_model_tables.cpp -- writes model_tables.inc, the frozen pair-model data
// of the library's bitstream qem-pair-v2 (spec S4).
//
// Page "Paired-count resident layout", "Operation pipeline" step 2: streams
// are coded with "a 1024-state tANS table from 32 Poisson pair models", and
// section "Contract": the coding parameters are fixed by the ABI string.  The
// models are therefore data of the format, not something each process may
// recompute: this program evaluates spec S4 once in IEEE double, in the order
// the spec writes it, and prints the integer results (pair frequencies, box
// sizes, selection costs) as C++ source.  The library compiles that output
// and does no floating-point work on the tables at run time, so another
// host's libm cannot change the bitstream.
//
// Build and run (host only, no GPU):
//   g++ -O2 -std=c++17 -o /tmp/gen_model_tables gen_model_tables.cpp
//   /tmp/gen_model_tables > model_tables.inc
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <vector>

namespace {

constexpr int kModels = 32;
constexpr int kStates = 1024;

struct Model {
    uint16_t freq[256];
    int box;
    uint32_t cost[16];
};

Model make_model(int m)
{
    Model out{};
    const double lambda = 0.005 * std::pow(3200.0, static_cast<double>(m) / 31.0);

    // Poisson(lambda) on 0..14 by the pmf recurrence; the tail is folded into 15.
    std::array<double, 16> q{};
    q[0] = std::exp(-lambda);
    for (int v = 1; v <= 14; ++v)
        q[v] = (q[v - 1] * lambda) / static_cast<double>(v);
    double head = 0.0;
    for (int v = 0; v <= 14; ++v)
        head += q[v];
    q[15] = std::max(0.0, 1.0 - head);

    // The box 0..A: the first A whose remaining mass is below 2^-20.
    int A = 15;
    for (int cand = 0; cand < 15; ++cand) {
        double rest = 0.0;
        for (int v = cand + 1; v <= 15; ++v)
            rest += q[v];
        if (rest < 1.0 / 1048576.0) {
            A = cand;
            break;
        }
    }
    out.box = A;

    double mass = 0.0;
    for (int v = 0; v <= A; ++v)
        mass += q[v];
    std::array<double, 16> t{};
    for (int v = 0; v <= A; ++v)
        t[v] = q[v] / mass;

    for (int v = 0; v < 16; ++v)
        out.cost[v] = v <= A ? static_cast<uint32_t>(std::floor(-256.0 * std::log2(t[v]) + 0.5)) : 0xFFFFFFFFu;

    // One reserved slot per box symbol, floor of the scaled product pmf, then
    // the leftover units to the largest fractional parts (lower symbol first).
    const double scale = static_cast<double>(kStates - (A + 1) * (A + 1));
    struct Cand {
        double frac;
        int sym;
    };
    std::vector<Cand> order;
    int used = 0;
    for (int s = 0; s < 256; ++s) {
        const int a = s & 15, b = s >> 4;
        if (a > A || b > A)
            continue;
        const double scaled = (t[a] * t[b]) * scale;
        const double whole = std::floor(scaled);
        out.freq[s] = static_cast<uint16_t>(1 + static_cast<int>(whole));
        used += out.freq[s];
        order.push_back({scaled - whole, s});
    }
    std::stable_sort(order.begin(), order.end(), [](const Cand &x, const Cand &y) { return x.frac > y.frac; });
    for (int k = 0; k < kStates - used; ++k)
        out.freq[order[k].sym] += 1;
    return out;
}

}  // namespace

int main()
{
    std::printf("// model_tables.inc -- frozen pair-model data of qem-pair-v2 (spec S4).\n"
                "// Written by gen_model_tables.cpp; do not edit by hand.\n"
                "// kFreq[m][a + 16 b]: tANS frequencies of pair (a, b), summing to 1024;\n"
                "// kBox[m]: largest count the model codes; kCost[m][v]: selection cost of\n"
                "// count v in 1/256 bit (0xFFFFFFFF outside the box).\n");
    Model all[kModels];
    for (int m = 0; m < kModels; ++m)
        all[m] = make_model(m);
    std::printf("static const uint16_t kFreq[%d][256] = {\n", kModels);
    for (int m = 0; m < kModels; ++m) {
        std::printf("    {");
        for (int s = 0; s < 256; ++s)
            std::printf("%s%u", s ? (s % 16 ? "," : ",\n     ") : "", all[m].freq[s]);
        std::printf("},\n");
    }
    std::printf("};\nstatic const uint8_t kBox[%d] = {", kModels);
    for (int m = 0; m < kModels; ++m)
        std::printf("%s%d", m ? "," : "", all[m].box);
    std::printf("};\nstatic const uint32_t kCost[%d][16] = {\n", kModels);
    for (int m = 0; m < kModels; ++m) {
        std::printf("    {");
        for (int v = 0; v < 16; ++v)
            std::printf("%s%uu", v ? "," : "", all[m].cost[v]);
        std::printf("},\n");
    }
    std::printf("};\n");
    return 0;
}
