// qmv_tc_plan.cuh -- compile-time plan that turns a thread's packed affine
// codes into 16-bit float PAIRS for the tensor-core path (host+device).
//
// A 16-bit float whose exponent field encodes 2^E (E = 7 for bf16, 10 for f16)
// and whose mantissa holds an integer field f at bits [s, s + fb) equals
// 2^E + f * 2^s exactly, as long as s + fb <= E.  Subtracting 2^E (one packed
// half-precision subtract per pair) leaves f * 2^s exactly.  One 32-bit value
// holds two such halves, so ONE masked OR builds two codes at once when the two
// fields sit at the right distance: the low field at bits [s_lo, s_lo + fb) and
// the high field at bits [16 + s_hi, 16 + s_hi + fb) of the same 32-bit window
// of the packed row (a funnel shift of two adjacent words picks the window).
//
// The plan pairs the fields of one "unit" (the bytes one thread loads): it
// repeatedly picks the window that pairs the most free fields (one shifted value
// then feeds several masked ORs); fields left without a partner use the low
// half only.  The factor
// 2^s of each field is taken out of x instead (x * 2^-s, exact for bf16 inputs,
// which share fp32's exponent range); for f16 inputs the plan keeps every field
// at its natural bit position (s = 0, or 4 for the high nibble of an 8-bit
// code), so x is used unscaled.
//
// 8-bit codes are decoded as two 4-bit fields (low nibble weight 1, high nibble
// weight 16): a bf16 mantissa has only 7 bits.
#pragma once

namespace qmv {

// Bytes / codes / fields of one thread's unit, per code width.
template <int B> struct TcGeom {
    static constexpr int FB = (B == 8) ? 4 : B;                                   // field bits
    static constexpr int UNIT_BYTES = (B == 2 || B == 4 || B == 8) ? 16 : 4 * B;  // one 16-byte load, or 32 codes
    static constexpr int UNIT_CODES = UNIT_BYTES * 8 / B;
    static constexpr int NF = UNIT_BYTES * 8 / FB;                                // fields per unit
    static constexpr int NW = UNIT_BYTES / 4;                                     // 32-bit words per unit
    static constexpr int SB = 4 * UNIT_CODES;                                     // codes per super-block (a quad's units)
};

struct TcPlanData {
    int np;                  // A registers (field pairs) per unit, rounded up to a multiple of 4
    int lo[64], hi[64];      // field index in the low / high half (-1: empty)
    int sh[64];              // window start: bit offset in the unit's LSB-first stream
    int slo[64], shi[64];    // field position inside its 16-bit half
};

// Code index (within the unit) and power-of-two weight exponent of field f.
template <int B> __host__ __device__ constexpr int tc_field_code(int f) { return B == 8 ? f / 2 : f; }
template <int B> __host__ __device__ constexpr int tc_field_wexp(int f) { return (B == 8 && (f & 1)) ? 4 : 0; }

template <int B, bool F16>
__host__ __device__ constexpr TcPlanData tc_make_plan() {
    using G = TcGeom<B>;
    TcPlanData P{};
    const int E = F16 ? 10 : 7;
    const int fb = G::FB, room = E - fb;
    const int bits = G::NF * fb;
    bool used[64] = {};
    int n = 0;
    // Fields that can sit in the low (hi == 0) or high (hi == 1) half of the
    // window starting at bit sh, and where.
    auto pos = [&](int f, int sh, int hi) -> int {
        const int s = fb * f - sh - 16 * hi;
        if (s < 0 || s > room) return -1;
        if (F16 && s != tc_field_wexp<B>(f)) return -1;
        return s;
    };
    // Repeatedly take the window that pairs the most free fields (a window at
    // a word boundary needs no shift and wins ties), pairing its low-fitting
    // fields with its high-fitting fields.
    for (int round = 0; round < 64; ++round) {
        int best_sh = -1, best_k = 0;
        for (int sh = 0; sh + 16 < bits; ++sh) {
            int nl = 0, nh = 0;
            for (int f = 0; f < G::NF; ++f) {
                if (used[f]) continue;
                if (pos(f, sh, 0) >= 0) ++nl;
                else if (pos(f, sh, 1) >= 0) ++nh;
            }
            const int k = nl < nh ? nl : nh;
            const int score = 2 * k + ((sh % 32) == 0 && k > 0 ? 1 : 0);
            if (score > 2 * best_k + (best_sh >= 0 && (best_sh % 32) == 0 ? 1 : 0)) { best_k = k; best_sh = sh; }
        }
        if (best_k == 0) break;
        int lo_f[8] = {}, hi_f[8] = {}, nl = 0, nh = 0;
        for (int f = 0; f < G::NF; ++f) {
            if (used[f]) continue;
            if (nl < 8 && pos(f, best_sh, 0) >= 0) lo_f[nl++] = f;
            else if (nh < 8 && pos(f, best_sh, 1) >= 0) hi_f[nh++] = f;
        }
        for (int q = 0; q < best_k; ++q) {
            P.lo[n] = lo_f[q]; P.hi[n] = hi_f[q]; P.sh[n] = best_sh;
            P.slo[n] = pos(lo_f[q], best_sh, 0); P.shi[n] = pos(hi_f[q], best_sh, 1);
            used[lo_f[q]] = used[hi_f[q]] = true;
            ++n;
        }
    }
    // Fields left over use the low half of their own window.
    for (int f = 0; f < G::NF; ++f) {
        if (used[f]) continue;
        int s = F16 ? tc_field_wexp<B>(f) : 0;
        if (s > fb * f) s = 0;
        P.lo[n] = f; P.hi[n] = -1; P.sh[n] = fb * f - s; P.slo[n] = s; P.shi[n] = 0;
        used[f] = true;
        ++n;
    }
    while (n & 3) { P.lo[n] = -1; P.hi[n] = -1; P.sh[n] = 0; P.slo[n] = 0; P.shi[n] = 0; ++n; }
    P.np = n;
    return P;
}

}  // namespace qmv
