// tables.cu -- the 32 Poisson pair models and their tANS tables (host side).
//
// Page "Paired-count resident layout", "Operation pipeline" step 2: each
// stream is coded with "a 1024-state tANS table from 32 Poisson pair models".
// The models and their quantisation are the library's spec S4; tANS is
// Duda's tabled asymmetric numeral systems (arXiv:1311.2540), with the spread
// of spec S5.  Page "Contract": the coding parameters are fixed by the ABI
// string.  So the S4 results (frequencies, box sizes, selection costs) are
// frozen integer data (model_tables.inc, written once by
// gen_model_tables.cpp) and everything derived here from them is integer
// arithmetic: no libm call can move a table from one host to another.
#include <array>
#include <mutex>

#include "qem_internal.h"

namespace qem {
namespace {

#include "model_tables.inc"

constexpr int kSpreadStep = 643;   // (5/8)L + 3, odd, so the walk covers all 1024 slots

int floor_log2(int y)
{
    int r = -1;
    while (y) {
        y >>= 1;
        ++r;
    }
    return r;
}

void make_model(int m, HostTables &T)
{
    // The model's frequencies, box and selection costs are the frozen S4 data.
    for (int s = 0; s < 256; ++s)
        T.freq[m][s] = kFreq[m][s];
    T.amax[m] = kBox[m];
    for (int v = 0; v < 16; ++v)
        T.cost[m][v] = kCost[m][v];

    // Spread symbols over the slots with the odd step, ascending symbol order.
    std::array<uint8_t, kStates> slot_sym{};
    int pos = 0;
    for (int s = 0; s < 256; ++s)
        for (int r = 0; r < T.freq[m][s]; ++r) {
            slot_sym[pos] = static_cast<uint8_t>(s);
            pos = (pos + kSpreadStep) % kStates;
        }

    // Decode entries (y = f + rank of the slot among its symbol's slots) and
    // the encoder's per-symbol slot lists in ascending slot order.
    std::array<int, 257> start{};
    for (int s = 0; s < 256; ++s)
        start[s + 1] = start[s] + T.freq[m][s];
    std::array<int, 256> seen{};
    for (int slot = 0; slot < kStates; ++slot) {
        const int s = slot_sym[slot];
        const int f = T.freq[m][s];
        const int y = f + seen[s];
        T.enc_slot[m][start[s] + seen[s]] = static_cast<uint16_t>(slot);
        ++seen[s];
        const int nb = 10 - floor_log2(y);
        const uint32_t newbase = static_cast<uint32_t>((y << nb) - kStates);
        T.dec[m][slot] = newbase | (static_cast<uint32_t>(nb) << 10) |
                         (static_cast<uint32_t>(s & 15) << 16) | (static_cast<uint32_t>(s >> 4) << 24);
    }
    for (int s = 0; s < 256; ++s) {
        const int f = T.freq[m][s];
        const uint32_t k0 = f ? static_cast<uint32_t>(10 - floor_log2(f)) : 0u;
        T.enc_sym[m][s] = static_cast<uint32_t>(f) | (static_cast<uint32_t>(start[s]) << 11) | (k0 << 22);
    }
}

// Runs of zero-bit (0,0) steps.  A slot whose symbol is (0,0) and whose
// entry reads no bits moves the decoder, deterministically, to slot newbase,
// which is strictly lower (newbase = f + rank - 1024 <= slot - (1024 - f)),
// so the runs follow from one ascending pass.  skip[slot] (16 bits): the run
// length from this slot, capped at 63, in bits 10-15, and the slot reached
// after that many steps in bits 0-9; 0 when the slot itself reads bits or
// carries another symbol.  A capped run continues from the slot it reaches.
void make_runs(int m, HostTables &T)
{
    std::array<int, kStates> run{}, next{};
    for (int slot = 0; slot < kStates; ++slot) {
        const uint32_t e = T.dec[m][slot];
        const uint32_t nb = (e >> 10) & 15u, sym = e >> 16, nx = e & 1023u;
        next[slot] = -1;
        if (sym == 0u && nb == 0u && nx < static_cast<uint32_t>(slot)) {
            next[slot] = static_cast<int>(nx);
            run[slot] = 1 + run[nx];
        }
    }
    if (m >= kRunModels)
        return;
    bool small = true;      // every count of the model's symbols fits 4 bits
    for (int slot = 0; slot < kStates; ++slot) {
        const int r = run[slot] < 63 ? run[slot] : 63;
        int at = slot;
        for (int k = 0; k < r; ++k)
            at = next[at];
        const uint32_t e = T.dec[m][at];
        const uint32_t a = (e >> 16) & 0xFFu, c = e >> 24;
        small = small && a < 16u && c < 16u;
        T.runs[m][slot] = (e & 1023u) | (((e >> 10) & 15u) << 10) | (static_cast<uint32_t>(r) << 14) |
                          ((a & 15u) << 20) | ((c & 15u) << 24) | (at != 0 ? 1u << 28 : 0u);
    }
    // decode by runs only where (0,0) holds at least 7/8 of the states (lambda
    // up to ~0.04 here), a prefix of the first kRunModels models; there a
    // stream needs ~15-40 events instead of 256 steps
    if (small && T.freq[m][0] >= 896 && (m == 0 || ((T.skip_models >> (m - 1)) & 1u)))
        T.skip_models |= 1u << m;
}

}  // namespace

const HostTables &host_tables()
{
    static HostTables tables;
    static std::once_flag once;
    std::call_once(once, [] {
        for (int m = 0; m < kModels; ++m)
            make_model(m, tables);
        tables.skip_models = 0u;
        for (int m = 0; m < kModels; ++m)
            make_runs(m, tables);
    });
    return tables;
}

}  // namespace qem
