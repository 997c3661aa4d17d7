// qmv_api.cu -- the C ABI of libqmv.so (declared in include/qmv.h): argument
// validation, the size-based kernel picker and the launches.
//
// The picker replaces the pages' three-way choice (MLX: qmv_fast when the
// input is aligned and N % 8 == 0, qmv_fast_rows when aligned and N % 8 != 0,
// a generic kernel otherwise -- MLX pull request "affine_qmv_fast_rows")
// with one kernel template whose launch shape is chosen from the sizes:
//   * path:   wide 16-byte chunk loads when K is a multiple of the wide chunk
//             and w_packed is 16-byte aligned, else 4-byte chunks (any K that
//             is a multiple of the group);
//   * rows:   rows per warp R (x reuse) grows with N; any N works (tail rows
//             are clamped and not stored), so there is no N % 8 cliff;
//   * split-K inside the block: for narrow N the K chunks of a row are spread
//             over up to 8 warps (wk) so one row still uses many threads;
//   * x tile: the K range staged in shared memory at a time.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/qmv.h"
#include "qmv_launch.cuh"
#include "qmv_tc_plan.cuh"
#include "qmv_umma.cuh"

namespace {

thread_local int g_last_cuda = 0;

struct Forced { int path = -1, R = -1, wk = -1, wr = -1; };
Forced g_forced;
std::atomic<int> g_test_skip{0};     // qmv_test_skip_last_copy

struct DevInfo { int sms = 0; int ok = 0; unsigned* fault = nullptr; };
DevInfo g_dev[64];
std::mutex g_dev_mu;

int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev[dev].ok) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
            cudaGetLastError();
            return 148;
        }
        g_dev[dev].sms = sms;
        g_dev[dev].ok = 1;
    }
    return g_dev[dev].sms;
}

int elem_bytes(int dtype) { return dtype == QMV_F32 ? 4 : 2; }

}  // namespace

// Fault word of the bulk-ring kernels: a bounded wait that expired ORs its
// code in (1: consumer, full stage; 2: producer, empty stage; 4: producer,
// own copies).  Zero at module load; read and cleared by qmv_device_fault.
__device__ unsigned g_qmv_fault;

namespace {

// Device address of g_qmv_fault on the current device (looked up once per
// device); nullptr if the lookup fails.
unsigned* fault_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { cudaGetLastError(); return nullptr; }
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev[dev].fault) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_qmv_fault) != cudaSuccess) { cudaGetLastError(); return nullptr; }
        g_dev[dev].fault = static_cast<unsigned*>(a);
    }
    return g_dev[dev].fault;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-format facts the picker needs (mirrors qmv::Fmt).
struct FmtInfo {
    int fam, bits, wide_units;
};

FmtInfo fmt_info(int fam, int bits) {
    int b = (fam == qmv::FAM_AFFINE || fam == qmv::FAM_SINT) ? bits
          : (fam == qmv::FAM_MXFP8 || fam == qmv::FAM_E4M3 || fam == qmv::FAM_E5M2) ? 8 : 4;
    int wu = b == 2 ? 4 : b == 3 ? 4 : b == 4 ? 2 : b == 5 ? 4 : b == 6 ? 2 : 1;
    return {fam, b, wu};
}

struct Plan {
    int maxm, R, wide, tc, npass, wk, wr, tile_iters, C;   // tc: 0 CUDA cores, 1 tensor cores, 2 + bulk ring
    int sps = 0, pitch = 0, spb = 1, sring = 0, soff = 0, boff = 0, sbw = 0;
    size_t smem;
    dim3 grid, block;
    qmv::UmmaParams um{};    // tc == 5: the tensor-memory kernel
    int mld = 0;
};

// Rows per warp on the wide path (x reuse vs registers); measured on B200:
// 4 rows win at M <= 2 for every width (5/6-bit included).
int rows_per_warp_cap(int bits, int maxm) {
    (void)bits;
    return maxm <= 2 ? 4 : 2;
}

// ---- tensor-core launch shape --------------------------------------------------
// Which path wins, measured on B200 (bf16 x): 6-bit codes have no field
// pairing (one mask per code), so the CUDA cores win there; with several x rows
// the tensor cores win (the CUDA cores would need M FMAs per code); with one x
// row they win only once the matrix is large enough to hide their longer
// pipeline (about 48 MB of packed weights).
bool tc_preferred(int M, int N, int K, int bits, int dtype) {
    if (N < 64 || bits == 6) return false;
    if (M >= 2) return true;
    if (bits == 8 || dtype != QMV_BF16) return false;   // one x row in f16 / f32: the CUDA cores win
    const double wbytes = (double)N * K * bits / 8.0;
    return wbytes >= 48.0 * 1024 * 1024;
}

template <int B> int tc_np() { return qmv::tc_make_plan<B, false>().np; }
int tc_np_of(int bits) {
    switch (bits) {
        case 2: return tc_np<2>(); case 3: return tc_np<3>(); case 4: return tc_np<4>();
        case 5: return tc_np<5>(); case 6: return tc_np<6>(); case 8: return tc_np<8>();
        default: return 0;
    }
}
int tc_unit_bytes(int bits) { return (bits == 2 || bits == 4 || bits == 8) ? 16 : 4 * bits; }

struct TcShape { int npass, wk, wr, tsb, sb; long long gx; size_t smem; };

bool tc_shape(int M, int N, int K, int bits, int G, int dtype, bool w16, TcShape* ts) {
    const int ub = tc_unit_bytes(bits);
    const int uc = ub * 8 / bits;
    const int SB = 4 * uc;
    if (K % SB != 0) return false;
    if (ub == 16 && !w16) return false;
    if (bits == 2 && G < 64) return false;          // a 64-code unit would span two groups
    const int segsz = G < SB ? G : SB;
    const int ngs = SB / segsz;
    const int cols = M * ngs;
    const int npass = cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : 0;
    if (npass == 0) return false;
    const int nsplit = dtype == QMV_BF16 ? 1 : dtype == QMV_F16 ? 2 : 3;
    const int np = tc_np_of(bits);
    const int nsbk = K / SB;
    const long long tiles = ((long long)N + 15) / 16;
    const int sms = device_sms();
    // about 8 warps per SM: split K over k-warps only when the 16-row tiles
    // alone cannot fill the GPU (measured best on B200 for 4..28K rows)
    const long long target = (long long)sms * 8;
    long long wk = 1;
    while (wk < 8 && tiles * wk < target) wk *= 2;
    if (wk > nsbk) wk = nsbk;
    if (wk < 1) wk = 1;
    long long wr = 8 / wk;
    if (wr > tiles) wr = tiles;
    if (wr < 1) wr = 1;
    if (g_forced.wk > 0) wk = g_forced.wk > 8 ? 8 : g_forced.wk;
    if (g_forced.wr > 0) wr = g_forced.wr;
    while (wk * wr > 8) --wr;
    const size_t red = (size_t)wk * wr * 16 * 8 * npass * 4;
    // per super-block of x tile: bf16 planes (x rows + zero row), sum(x) and
    // sum(x~) per segment, two per-unit sums
    const size_t per_sb = (size_t)nsplit * (M + 1) * 4 * np * 4 + (size_t)M * ngs * 4 * 2 + (size_t)M * 4 * 2 * 4;
    const size_t fixed = (size_t)nsplit * (M + 1) * 16 + red;
    const size_t budget = 160 * 1024;
    long long tsb = budget > fixed ? (long long)((budget - fixed) / per_sb) : 0;
    if (tsb > nsbk) tsb = nsbk;
    if (tsb < 1) return false;
    ts->npass = npass; ts->wk = (int)wk; ts->wr = (int)wr; ts->tsb = (int)tsb; ts->sb = SB;
    ts->gx = (tiles + wr - 1) / wr;
    ts->smem = (size_t)nsplit * (M + 1) * ((size_t)tsb * 4 * np + 4) * 4 + (size_t)M * tsb * ngs * 4 * 2 +
               (size_t)M * tsb * 4 * 2 * 4 + red;
    return ts->gx <= 0x7FFFFFFFLL && ts->smem <= (size_t)qmv::kMaxSmem;
}

// ---- per-group tensor-core ring launch shape (qmv_tcg.cuh) ----------------------
// 4-bit codes, bf16 / f16 x, G in {32, 64, 128}, K a multiple of 8 groups (a
// ring stage is 8 groups; the scale tiles' tensor maps need 16-byte row
// strides), up to 32 x rows (nt n-tiles of 8).  Row blocks of 16 * wr rows over
// a persistent grid, wk in {1, 2, 4, 8} k-warps, 8 to 16 consumer warps.  Shared
// memory: a ring of about 72 KB (2..8 stages), x staged for the whole K when it
// fits beside a ring of at least 3 stages, else in tiles of whole stages.
// The shape minimises, measured on B200 (M = 8, the 7B layer's projections):
//   rounds of row blocks over the SMs x rows per block
//   x (1 + log2(wk) / 4)     (a k-warp's fixed cost per stage: fewer, longer
//                              k-ranges win once the SMs are busy)
//   x 1.25 below 12 consumer warps (more warps hide more latency)
//   x rounds again when x is tiled (staged anew for every row block)
struct TcgShape { int nt, wk, wr, nst, sby, xt; long long gx; size_t smem; };

bool tcg_plan_smem(int nt, int wk, int wr, int K, int G, TcgShape* ts) {
    const int nc = 8 * nt;
    const int rows = 16 * wr;
    const int sby = ((rows * (4 * G + 32) + 1023) / 1024) * 1024;      // codes + scale and bias tiles
    int nst = (72 * 1024) / sby;
    nst = nst < 2 ? 2 : (nst > 8 ? 8 : nst);
    const long long nks = K / (8 * G);
    const size_t red = (size_t)(wr * wk) * 16 * nc * 4;
    const size_t per_stage_x = (size_t)(G / 2) * nt * 32 * 8 + (size_t)8 * nc * 4;
    const size_t lim = (size_t)qmv::kMaxSmem;
    const size_t whole = 2048 + red + (size_t)nks * per_stage_x;
    long long xt;
    if (whole + 3 * (size_t)sby <= lim) {
        const long long fit = (long long)((lim - whole) / sby);
        if (fit < nst) nst = (int)fit;
        xt = nks;
    } else {
        const size_t fixed = 2048 + red + (size_t)nst * sby;
        if (fixed + per_stage_x > lim) return false;
        xt = (long long)((lim - fixed) / per_stage_x);
        if (xt > nks) xt = nks;
    }
    ts->nt = nt; ts->wk = wk; ts->wr = wr; ts->nst = nst; ts->sby = sby; ts->xt = (int)xt;
    ts->smem = 2048 + (size_t)nst * sby + (size_t)xt * per_stage_x + red;
    return ts->smem <= lim;
}

bool tcg_shape(int M, int N, int K, int bits, int G, int dtype, bool w16, bool s16, TcgShape* ts) {
    if (bits != 4 || (dtype != QMV_BF16 && dtype != QMV_F16)) return false;
    if (G != 32 && G != 64 && G != 128) return false;
    if (M < 1 || M > 32 || N < 1 || K <= 0 || K % (8 * G) != 0 || !w16 || !s16) return false;
    const int nt = M <= 8 ? 1 : M <= 16 ? 2 : 4;
    const int sms = device_sms();
    const long long nks = K / (8 * G);
    double best = -1.0;
    for (int wk = 1; wk <= 8; wk *= 2) {
        for (int wr = 1; wr * wk <= 16; ++wr) {
            const int ncw = wr * wk;
            if (ncw < 8) continue;
            if (g_forced.wr > 0 && wr != g_forced.wr) continue;
            if (g_forced.wk > 0 && wk != g_forced.wk) continue;
            TcgShape t;
            if (!tcg_plan_smem(nt, wk, wr, K, G, &t)) continue;
            const long long nrb = ((long long)N + 16 * wr - 1) / (16 * wr);
            const long long rounds = (nrb + sms - 1) / sms;
            const int lg = wk == 1 ? 0 : wk == 2 ? 1 : wk == 4 ? 2 : 3;
            double cost = (double)rounds * wr * (1.0 + 0.25 * lg) * (ncw < 12 ? 1.25 : 1.0);
            if (t.xt < nks) cost *= (double)rounds;
            if (best < 0 || cost < best) {
                best = cost;
                *ts = t;
                ts->gx = nrb < sms ? nrb : sms;
            }
        }
    }
    return best >= 0;
}

// ---- bulk-ring tensor-core launch shape ----------------------------------------
// Row blocks of 16*wr rows are spread over a persistent grid of one block per
// SM, wk = 8 / wr consumer warps split K.  A ring stage holds about 32 KB;
// the x tile takes what shared memory is left.
struct TcbShape { int npass, spb, wk, wr, tsb, sps, pitch, sring, soff, boff, sbw; long long gx; size_t smem; };

bool tcb_shape(int M, int N, int K, int bits, int G, int dtype, bool w16, bool s16, TcbShape* ts) {
    const int ub = tc_unit_bytes(bits);
    const int uc = ub * 8 / bits;
    const int SB = 4 * uc;
    if (K % SB != 0 || !w16) return false;
    if (((long long)K * bits / 8) % 16 != 0) return false;     // bulk copies: 16-byte rows
    if (bits == 2 && G < 64) return false;
    const int segsz = G < SB ? G : SB;
    const int ngs = SB / segsz;
    const int cols = M * ngs;
    const int npass = cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : 0;
    if (npass == 0) return false;
    int spb = 8 * npass / cols;
    spb = spb >= 8 ? 8 : spb >= 4 ? 4 : spb >= 2 ? 2 : 1;
    const int nsplit = dtype == QMV_BF16 ? 1 : dtype == QMV_F16 ? 2 : 3;
    const int es = elem_bytes(dtype);
    const int np = tc_np_of(bits);
    const int nsbk = K / SB;
    const int sms = device_sms();
    // Consumer warps and rows per block (measured on B200).  One x row: 8
    // consumer warps, 32-row blocks (2-bit: 64).  Several x rows: 12 consumer
    // warps, wr in {2, 3, 4} (wk = 12 / wr) minimising (rounds of row blocks
    // over the SMs) x (rows per block), i.e. the busiest SM's share.
    // x of the whole K staged once per block needs about this much shared memory
    const long long x_bytes = (long long)nsplit * M * (K / uc) * np * 4;
    int wr, wk;
    if (M == 1 || (N >= 15360 && (M == 2 || x_bytes > 96 * 1024))) {
        // one or two x rows over many rows, or x too large to stay staged
        // across row blocks: 128-row blocks, K not split, as few row blocks
        // per block as possible (5-bit: 64 rows, K over 2 warps)
        // (one scale group per super-block, ngs = 1: only SPB slot columns of 8
        // are live, so 64-row blocks with K over 2 warps measured faster too)
        wr = (bits == 5 || ngs == 1) ? 4 : 8;
        wk = 8 / wr;
    } else {
        wr = 2;
        long long best = -1;
        for (int w = 2; w <= 4; ++w) {
            const long long nrb = ((long long)N + 16 * w - 1) / (16 * w);
            const long long cost = ((nrb + sms - 1) / sms) * w;
            if (best < 0 || cost < best) { best = cost; wr = w; }
        }
        wk = 12 / wr;
    }
    if (g_forced.wr > 0) wr = g_forced.wr > 12 ? 12 : g_forced.wr;
    if (g_forced.wk > 0) wk = g_forced.wk > 12 ? 12 : g_forced.wk;
    if (wk > nsbk) wk = nsbk;
    if (wk < 1) wk = 1;
    // a block is 8 or 12 consumer warps: otherwise the largest wk <= the
    // chosen one that divides such a count, and its wr
    auto valid_ncw = [&](int n) { return n == 8 || n == 12; };
    if (!valid_ncw(wk * wr)) {
        int bk = 0, bw = 0;
        for (int k = wk; k >= 1 && bk == 0; --k)
            for (int n = 8; n <= 12 && bk == 0; n += 4)
                if (valid_ncw(n) && n % k == 0) { bk = k; bw = n / k; }
        wk = bk; wr = bw;
    }
    const int rows = 16 * wr;
    // stage size: a multiple of one batch of every k-warp (SPB * wk super-blocks)
    // and of the super-blocks one group spans (G / SB when G > SB)
    const int gq = G > SB ? G / SB : 1;
    auto quantum_of = [&](int b) { int qv = b * wk; while (qv % gq) qv *= 2; return qv; };
    // a ring stage of one quantum must leave room for the x tile: fewer
    // super-blocks per batch (fewer slot columns used) where it would not
    while (spb > 1 && (size_t)qmv::kTcbStages * rows * quantum_of(spb) * 4 * ub > 144 * 1024) spb /= 2;
    const int quantum = quantum_of(spb);
    // scale bytes of s super-blocks (G <= SB: s * SB / G groups; else s / (G / SB))
    int sps = 32768 / (rows * 4 * ub);
    sps = sps / quantum * quantum;
    if (sps < quantum) sps = quantum;
    if (sps > nsbk) sps = (nsbk + quantum - 1) / quantum * quantum;
    if (rows > 256) return false;
    // a scale tile row must be a whole number of 16 bytes to travel in the
    // ring: grow a short stage to the next such multiple of the quantum
    if (s16 && ((long long)(K / G) * es) % 16 == 0) {
        auto sb_bytes = [&](int v) { return (G <= SB ? v * (SB / G) : v / (G / SB)) * es; };
        int v = sps;
        while (v < 4 * sps && v < nsbk && sb_bytes(v) % 16 != 0) v += quantum;
        if (sb_bytes(v) % 16 == 0 && v * 4 * ub / 8 <= 256) sps = v;
    }
    while (sps > quantum && sps * 4 * ub / 8 > 256) sps -= quantum;
    if (sps * 4 * ub / 8 > 256) return false;
    // stage layout: ROWS packed rows of pitch = S * 4 * UB bytes, then (scales
    // in the ring) a scale tile and a bias tile of ROWS x sbw bytes; each is
    // one tensor copy, whose column start must sit on 16 bytes and whose box
    // is at most 256 elements a side (the rows' box counts 8-byte elements)
    auto layout = [&](int s, int* sring, int* sbw, int* stage) {
        const int box0 = G <= SB ? s * (SB / G) : s / (G / SB);
        *sbw = box0 * es;
        *sring = (s16 && ((long long)(K / G) * es) % 16 == 0 && *sbw % 16 == 0 && box0 <= 256 && rows <= 256) ? 1 : 0;
        const int pitch = s * 4 * ub;                 // dense rows, as the tensor copy lays them out
        *stage = rows * pitch + (*sring ? 2 * rows * *sbw : 0);
        return pitch;
    };
    const int ncw = wk * wr;
    const size_t red = (size_t)ncw * 16 * 8 * npass * 4;
    const size_t per_sb = (size_t)nsplit * M * 4 * np * 4 + (size_t)M * ngs * 4 * 2 + (size_t)M * 4 * 2 * 4;
    long long tsb = 0;
    int sring = 0, sbw = 0, stage = 0, pitch = 0;
    for (;;) {
        pitch = layout(sps, &sring, &sbw, &stage);
        // 128 bytes of barriers + 128 of alignment slack for the ring
        const size_t fixed = 256 + (size_t)qmv::kTcbStages * stage + red + (size_t)nsplit * (M * 4 + 4 * np + 4) * 4;
        tsb = fixed < (size_t)qmv::kMaxSmem ? (long long)(((size_t)qmv::kMaxSmem - fixed) / per_sb) : 0;
        if (tsb >= nsbk) { tsb = nsbk; break; }
        tsb = tsb / sps * sps;
        if (tsb >= sps) break;
        if (sps <= quantum) return false;
        sps = (sps / 2) / quantum * quantum;
        if (sps < quantum) sps = quantum;
    }
    const long long nrb = ((long long)N + rows - 1) / rows;
    ts->npass = npass; ts->spb = spb; ts->wk = wk; ts->wr = wr; ts->tsb = (int)tsb; ts->sps = sps;
    ts->pitch = pitch; ts->sring = sring; ts->sbw = sbw;
    ts->soff = rows * pitch; ts->boff = rows * pitch + rows * sbw;
    ts->gx = nrb < sms ? nrb : sms;
    const size_t plane = (size_t)M * ((size_t)tsb * 4 * np + 4) + 4 * np + 4;
    ts->smem = 256 + (size_t)qmv::kTcbStages * stage + (size_t)nsplit * plane * 4 +
               (size_t)M * tsb * ngs * 4 * 2 + (size_t)M * tsb * 4 * 2 * 4 + red;
    return ts->smem <= (size_t)qmv::kMaxSmem;
}

// ---- CUDA-core ring launch shape (one bf16 x row, qmv_tcf.cuh) ---------------
// Same ring and stage layout as the tensor-core ring; a warp takes two
// super-blocks per step, so a stage is a multiple of 2 * wk super-blocks.  The
// x tile holds (NP + 4) words of x~ pairs and two sums per unit (affine), or
// UC + 4 fp32 x values per unit (fp: the block-scaled FP formats, whose
// scales stay in global memory).
bool tcf_shape(int N, int K, int bits, int G, bool w16, bool s16, TcbShape* ts, bool fp = false, int fp_es = 1) {
    const int ub = tc_unit_bytes(bits);
    const int uc = ub * 8 / bits;
    const int SB = 4 * uc;
    if (K % SB != 0 || !w16) return false;
    if (((long long)K * bits / 8) % 16 != 0) return false;     // tensor copies: 16-byte rows
    if (!fp && G < uc) return false;                            // a unit lies in one group
    // scale elements: affine 2 bytes (the ring serves bf16 x); FP: the
    // format's block-scale bytes, one tile per stage (no biases)
    const int es = fp ? fp_es : 2;
    const int ntiles = fp ? 1 : 2;
    const int nps = fp ? uc + 4 : tc_np_of(bits) + 4;
    const int nsbk = K / SB;
    const int sms = device_sms();
    // Block shape (measured on B200): the fewest rows on the busiest SM
    // (rounds of row blocks over the SMs x rows per block), with at least 4
    // steps of 2 super-blocks per warp and row block; ties go to 8 compute
    // warps, then to fewer row blocks.
    const int steps = (nsbk + 1) / 2;
    int wr = 8, wk = 1;
    {
        static const int cand[10][2] = {{8, 1}, {4, 2}, {2, 4}, {1, 8},
                                        {12, 1}, {6, 2}, {4, 3}, {3, 4}, {2, 6}, {1, 12}};
        long long best = -1;
        for (const auto& c : cand) {
            const int k = c[0], r = c[1];
            if (k > 1 && steps < 4 * k) continue;
            const long long nrb_c = ((long long)N + 16 * r - 1) / (16 * r);
            const long long cost = ((nrb_c + sms - 1) / sms) * 16 * r;
            const bool same_warps = (k * r) == (wk * wr);
            if (best < 0 || cost < best || (cost == best && same_warps && r > wr)) { best = cost; wk = k; wr = r; }
        }
    }
    if (g_forced.wr > 0) wr = g_forced.wr > 12 ? 12 : g_forced.wr;
    if (g_forced.wk > 0) wk = g_forced.wk > 12 ? 12 : g_forced.wk;
    const int ncw = wk * wr;
    if (ncw != 8 && ncw != 12) return false;
    const int rows = 16 * wr;
    const int gq = G > SB ? G / SB : 1;
    int quantum = 2 * wk;
    while (quantum % gq) quantum *= 2;
    int sps = 32768 / (rows * 4 * ub);
    sps = sps / quantum * quantum;
    if (sps < quantum) sps = quantum;
    if (sps > nsbk) sps = (nsbk + quantum - 1) / quantum * quantum;
    if (s16 && ((long long)(K / G) * es) % 16 == 0) {
        auto sb_bytes = [&](int v) { return (G <= SB ? v * (SB / G) : v / (G / SB)) * es; };
        int v = sps;
        while (v < 4 * sps && v < nsbk && sb_bytes(v) % 16 != 0) v += quantum;
        if (sb_bytes(v) % 16 == 0 && v * 4 * ub / 8 <= 256) sps = v;
    }
    while (sps > quantum && sps * 4 * ub / 8 > 256) sps -= quantum;
    if (sps * 4 * ub / 8 > 256) return false;
    auto layout = [&](int s, int* sring, int* sbw, int* stage) {
        const int box0 = G <= SB ? s * (SB / G) : s / (G / SB);
        *sbw = box0 * es;
        *sring = (s16 && ((long long)(K / G) * es) % 16 == 0 && *sbw % 16 == 0 && box0 <= 256 && rows <= 256) ? 1 : 0;
        const int pitch = s * 4 * ub;
        *stage = rows * pitch + (*sring ? ntiles * rows * *sbw : 0);
        return pitch;
    };
    const size_t red = (size_t)(qmv::kTcbStages + 1) * ncw * 16 * 4;
    const size_t per_sb = (size_t)4 * (nps * 4 + (fp ? 0 : 8));
    long long tsb = 0;
    int sring = 0, sbw = 0, stage = 0, pitch = 0;
    for (;;) {
        pitch = layout(sps, &sring, &sbw, &stage);
        const size_t fixed = 256 + (size_t)qmv::kTcbStages * stage + red;
        tsb = fixed < (size_t)qmv::kMaxSmem ? (long long)(((size_t)qmv::kMaxSmem - fixed) / per_sb) : 0;
        if (tsb >= nsbk) { tsb = nsbk; break; }
        tsb = tsb / sps * sps;
        if (tsb >= sps) break;
        if (sps <= quantum) return false;
        sps = (sps / 2) / quantum * quantum;
        if (sps < quantum) sps = quantum;
    }
    const long long nrb = ((long long)N + rows - 1) / rows;
    ts->npass = 0; ts->spb = 1; ts->wk = wk; ts->wr = wr; ts->tsb = (int)tsb; ts->sps = sps;
    ts->pitch = pitch; ts->sring = sring; ts->sbw = sbw;
    ts->soff = rows * pitch; ts->boff = rows * pitch + rows * sbw;
    ts->gx = nrb < sms ? nrb : sms;
    ts->smem = 256 + (size_t)qmv::kTcbStages * stage + (size_t)tsb * per_sb + red;
    return ts->smem <= (size_t)qmv::kMaxSmem;
}

// ---- tensor-memory (tcgen05) launch shape (qmv_umma.cuh) ---------------------
// Geometry per code width (mirrors qmv::UmGeom).
struct UmGeomH { int uc, npu, slot_cols, stage_codes, stage_bytes; };
template <int B> UmGeomH um_geom_t() {
    using G = qmv::UmGeom<B>;
    return {G::UC, G::NPU, G::SLOT_COLS, G::STAGE_CODES, G::STAGE_BYTES};
}
bool um_geom(int bits, UmGeomH* g) {
    switch (bits) {
        case 2: *g = um_geom_t<2>(); return true;
        case 3: *g = um_geom_t<3>(); return true;
        case 4: *g = um_geom_t<4>(); return true;
        case 5: *g = um_geom_t<5>(); return true;
        case 6: *g = um_geom_t<6>(); return true;
        case 8: *g = um_geom_t<8>(); return true;
        default: return false;
    }
}
long long gcd_ll(long long a, long long b) { while (b) { long long t = a % b; a = b; b = t; } return a; }

// Clusters of S CTAs (one per SM) that fit at once, per device (queried once).
int um_clusters(int bits, const qmv::UmmaParams& u, size_t smem) {
    static int cache[64][17] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { cudaGetLastError(); return 1; }
    std::lock_guard<std::mutex> lk(g_dev_mu);
    int& c = cache[dev][u.S];
    if (!c) {
        int n = 0;
        if (qmv::umma_max_clusters(bits, u, smem, &n) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = device_sms() / u.S;
        }
        c = n < 1 ? 1 : n;
    }
    return c;
}

// Affine, bf16 x, one weight matrix, M <= 64.  Rows: 128-row tiles over a
// persistent grid of clusters; K split over the S CTAs of a cluster when the
// tiles alone leave SMs idle, or when x of the whole K would not fit.
bool umma_shape(int M, int N, int K, int bits, int G, int dtype, bool w16, bool s16, bool x16, int batch, Plan* pl) {
    UmGeomH g;
    if (!um_geom(bits, &g)) return false;
    if (dtype != QMV_BF16 || batch != 1 || M < 1 || M > 64 || N < 1 || K < 64) return false;
    if (!w16 || !s16 || !x16) return false;
    if (G < g.uc || K % 64 != 0 || K % G != 0 || (K / G) % 8 != 0) return false;
    if (((long long)K * bits / 8) % 16 != 0) return false;
    const int BLK = G > 64 ? G : 64, NBG = BLK / G, NBS = BLK / 64;
    int mld = 1;
    while (mld < M) mld *= 2;
    const int ncol = mld < 16 ? 16 : mld;                          // MMA N >= the accumulator read width
    const int blk_cols = NBS * g.slot_cols + NBG * ncol;
    int DB = 2 * (512 / (2 * blk_cols));
    if (DB > 16) DB = 16;
    if (DB < 2) return false;
    const long long QC = (long long)g.stage_codes / gcd_ll(g.stage_codes, 8LL * G) * (8LL * G);
    const int nq = (int)((K + QC - 1) / QC);
    const int tiles = (N + 127) / 128;
    const int ksg = 2 * g.npu * G / g.uc;                       // k-slots per group
    const int SSL = G == 32 ? 8 : 4;                             // scale slots: 8 groups each
    auto smem_of = [&](int S, int WST, unsigned* smem_b) {
        const long long rng = std::min<long long>((long long)((nq + S - 1) / S) * QC, K);
        const long long ngr = rng / G;
        *smem_b = (unsigned)(ngr * ksg * M * 2 + 1024);
        return (size_t)2048 + (size_t)WST * g.stage_bytes + (size_t)SSL * 4096 + *smem_b + (size_t)(M * ngr + 3) / 4 * 16 +
               (size_t)DB * NBG * 128 * 8 + (size_t)128 * mld * 4;
    };
    const int smax = std::min(16, nq);       // clusters beyond 8 are non-portable; B200 takes 16
    int S = 0, WST = 0;
    unsigned sb = 0;
    for (int s_ = 1; s_ <= smax && !S; ++s_)
        for (int w = 4; w >= 2; --w)
            if (smem_of(s_, w, &sb) <= (size_t)qmv::kMaxSmem) { S = s_; WST = w; break; }
    if (!S) return false;
    const int sms = device_sms();
    if (tiles < sms) {
        int so = sms / tiles;
        if (so > smax) so = smax;
        if (so > S) S = so;
    }
    if (g_forced.wk > 0 && g_forced.wk <= smax) S = g_forced.wk;       // test knob: the K split
    WST = 0;
    for (int w = 4; w >= 2; --w)
        if (smem_of(S, w, &sb) <= (size_t)qmv::kMaxSmem) { WST = w; break; }
    if (!WST) return false;
    size_t smem = smem_of(S, WST, &sb);
    if (smem < 120 * 1024) smem = 120 * 1024;                      // one CTA per SM
    qmv::UmmaParams& u = pl->um;
    u.S = S; u.DB = DB; u.WST = WST; u.SSL = SSL; u.nq = nq; u.QC = (int)QC; u.ncols = 512; u.ncol_mma = ncol;
    u.tiles = tiles; u.smem_b = sb;
    u.ngr_max = (int)(std::min<long long>((long long)((nq + S - 1) / S) * QC, K) / G);
    int ncl = um_clusters(bits, u, smem);
    if (ncl > tiles) ncl = tiles;
    pl->maxm = M; pl->R = 1; pl->wide = 1; pl->tc = 5; pl->npass = 0; pl->wk = S; pl->wr = 1;
    pl->tile_iters = DB; pl->C = BLK; pl->smem = smem; pl->mld = mld;
    pl->grid = dim3((unsigned)S, (unsigned)ncl, 1);
    pl->block = dim3(320, 1, 1);
    return true;
}

// The per-group tensor-core ring for automatic plans: from 8 x rows (qmm
// chunks up to 32), and from 4 for tall matrices.  Measured on B200 (4-bit g64
// bf16, the 7B layer's projections, back-to-back calls): at M = 8 against the
// tensor-core ring QKV 10.7 / 13.3 us, O 9.5 / 11.3, gate+up 26.3 / 44.1, down
// 29.8 / 30.9; qmm M = 16..64 1.6-3x faster than the tensor-memory kernel or
// the ring's chunks; at M = 4 gate+up 25.3 / 32.6 us, but the smaller shapes
// stay faster on the ring below 8 rows (x is staged as 8 rows whatever M).
bool tcg_preferred(int M, int N, int bits) {
    return bits == 4 && M <= 32 && (M >= 8 || (M >= 4 && N >= 20000));
}

// Choose the launch shape.  Returns QMV_OK or an error (sizes too large).
int make_plan(int fam, int M, int N, int K, int bits, int G_of_plan, int dtype, bool w16, int batch, Plan* pl,
              bool s16 = true, bool gather = false, bool pair = false, bool x16 = true, bool qmm = false,
              bool qkv = false, bool norm = false, int fp_es = 1) {
    // pair (fused gate + up): N counts the 2N virtual rows; pair, Q / K / V
    // and the fused RMSNorm run on the row-tiled CUDA-core kernel only
    if (pair || qkv || norm) gather = true;
    const FmtInfo fi = fmt_info(fam, bits);
    const bool aff = fam == qmv::FAM_AFFINE;                 // the affine-only kernels
    const bool affl = aff || fam == qmv::FAM_SINT;           // sum(x) staged with x
    int maxm = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
    const int c_wide = 32 * fi.wide_units;
    bool wide = w16 && (K % c_wide == 0);
    if (g_forced.path == 0) wide = false;

    // ---- few output rows: the latency kernel (weights dequantized before the
    // grid-dependency wait, one block per row) --------------------------------
    // (N <= 64 any M; up to 512 rows for one or two x rows: measured faster
    // than the row-tiled kernels on B200 up to about 1.3 MB of weights)
    if (!pair && !qkv && !norm && K > 0 &&
        (g_forced.path == 5 || (g_forced.path < 0 && (N <= 64 || (N <= 512 && M <= 2))))) {
        const int units = K / 32;
        int thr = ((units + 31) / 32) * 32;
        if (thr > 256) thr = 256;
        if (thr < 32) thr = 32;
        const long long row_bytes = (long long)K * fi.bits / 8;
        pl->maxm = maxm; pl->R = 1; pl->tc = 3; pl->npass = 0; pl->wk = thr / 32; pl->wr = 1;
        pl->wide = (w16 && fi.bits % 4 == 0 && row_bytes % 16 == 0) ? 1 : 0;
        pl->tile_iters = (units + thr - 1) / thr; pl->C = 32; pl->smem = (size_t)8 * maxm * 4;
        pl->grid = dim3((unsigned)N, 1, (unsigned)batch);
        pl->block = dim3((unsigned)thr, 1, 1);
        return QMV_OK;
    }

    // ---- tensor-memory kernel (tcgen05) ---------------------------------------
    // Measured on B200: one tcgen05.mma kind::f16 (M = 128, K = 16) takes about
    // 191 cycles whatever N is (16..256), so the tensor cores take in at most
    // 128 * 16 / 191 = 10.7 weights per cycle per SM (about 1.6 TB/s of 4-bit
    // weights): below the other kernels for M <= 8.  For x rows beyond 8 (qmm)
    // it decodes every weight once where chunks decode it once per chunk; qmm
    // takes it for matrices of few row tiles (qmm_prefers_umma).
    if (!gather && aff && K > 0 && (g_forced.path == 7 || qmm) &&
        umma_shape(M, N, K, bits, G_of_plan, dtype, w16, s16, x16, batch, pl))
        return QMV_OK;

    // ---- one bf16 x row: CUDA cores with the weight ring ----------------------
    // (measured on B200: the fastest path for one bf16 x row from about 10 MB
    // of 2/3/4/5/6-bit weights; 8-bit codes take two fields each, and there
    // the register-streaming CUDA-core kernel is as fast)
    // The block-scaled FP formats take the same ring, their block scales
    // copied into each stage next to the codes.  Measured on B200 (M = 1,
    // bf16, 8192^2 .. 16384^2 and the layer shapes): the ring wins for
    // FP32- and FP16-scaled formats (NVFP8 16384^2 110 -> 95 us, 28672 x
    // 4096 63 -> 44 us; FP4_F16 80 -> 63 us), where the row-tiled kernel's
    // per-chunk scale loads weigh most, and loses a little for the
    // byte-scaled ones (MXFP8-E4M3 16384^2 63 -> 66 us), which stay row-tiled.
    const bool fp_fam = fam == qmv::FAM_MXFP4 || fam == qmv::FAM_NVFP4 || fam == qmv::FAM_MXFP8 ||
                        fam == qmv::FAM_E2M1 || fam == qmv::FAM_E4M3 || fam == qmv::FAM_E5M2;
    const bool big = (double)N * K * fi.bits / 8.0 >= 10.0 * 1024 * 1024;
    const bool fma_ring_pick = M == 1 && dtype == QMV_BF16 && big &&
                               (aff ? (bits >= 2 && bits <= 6) : (fp_fam && fp_es >= 2));
    if (!gather && (aff || fp_fam) && K > 0 && M == 1 && dtype == QMV_BF16 &&
        (g_forced.path == 6 || (g_forced.path < 0 && fma_ring_pick))) {
        TcbShape ts;
        if (tcf_shape(N, K, fi.bits, G_of_plan, w16, s16, &ts, !aff, fp_es)) {
            pl->maxm = 1; pl->R = 1; pl->wide = 1; pl->tc = 4; pl->npass = 0;
            pl->wk = ts.wk; pl->wr = ts.wr; pl->tile_iters = ts.tsb; pl->sps = ts.sps; pl->pitch = ts.pitch;
            pl->spb = 1; pl->sring = ts.sring; pl->soff = ts.soff; pl->boff = ts.boff; pl->sbw = ts.sbw;
            pl->C = 4 * tc_unit_bytes(fi.bits) * 8 / fi.bits; pl->smem = ts.smem;
            pl->grid = dim3((unsigned)ts.gx, 1, (unsigned)batch);
            pl->block = dim3(32 * (ts.wk * ts.wr + 1), 1, 1);
            return QMV_OK;
        }
    }

    // ---- per-group tensor-core ring kernel (4-bit, bf16 / f16, M <= 32) --------
    if (!gather && aff && K > 0 && (g_forced.path == 8 || (g_forced.path < 0 && tcg_preferred(M, N, bits)))) {
        TcgShape ts;
        if (tcg_shape(M, N, K, bits, G_of_plan, dtype, w16, s16, &ts)) {
            pl->maxm = 8 * ts.nt; pl->R = 1; pl->wide = 1; pl->tc = 6; pl->npass = ts.nt;
            pl->wk = ts.wk; pl->wr = ts.wr; pl->tile_iters = ts.xt; pl->sps = ts.nst; pl->pitch = ts.sby;
            pl->spb = 1; pl->sring = 1; pl->soff = 0; pl->boff = 0; pl->sbw = 16;
            pl->C = G_of_plan; pl->smem = ts.smem;
            pl->grid = dim3((unsigned)ts.gx, 1, (unsigned)batch);
            pl->block = dim3(32 * (ts.wk * ts.wr + 1), 1, 1);       // + the producer warp
            return QMV_OK;
        }
    }

    // ---- tensor-core kernel with the bulk-copy weight ring --------------------
    // (measured on B200: the fastest path once M >= 2, and for large 2/3/4/5-bit
    // matrices at M = 1)
    // (6-bit codes do not pair: the ring kernel wins there only at M = 8)
    const bool ring_pick = M >= 2 ? (N >= 64 && (bits != 6 || M >= 8)) : tc_preferred(M, N, K, bits, dtype);
    if (!gather && aff && K > 0 && (g_forced.path == 4 || (g_forced.path < 0 && ring_pick))) {
        TcbShape ts;
        if (tcb_shape(M, N, K, bits, G_of_plan, dtype, w16, s16, &ts)) {
            pl->maxm = maxm; pl->R = 1; pl->wide = 1; pl->tc = 2; pl->npass = ts.npass;
            pl->wk = ts.wk; pl->wr = ts.wr; pl->tile_iters = ts.tsb; pl->sps = ts.sps; pl->pitch = ts.pitch;
            pl->spb = ts.spb; pl->sring = ts.sring; pl->soff = ts.soff; pl->boff = ts.boff; pl->sbw = ts.sbw;
            pl->C = 4 * tc_unit_bytes(bits) * 8 / bits; pl->smem = ts.smem;
            pl->grid = dim3((unsigned)ts.gx, 1, (unsigned)batch);
            pl->block = dim3(32 * (ts.wk * ts.wr + 1), 1, 1);       // + the producer warp
            return QMV_OK;
        }
    }

    // ---- tensor-core kernel (affine, enough rows to fill the GPU) -------------
    if (!gather && aff && K > 0 && g_forced.path != 0 && g_forced.path != 1 &&
        (g_forced.path == 3 || tc_preferred(M, N, K, bits, dtype))) {
        TcShape ts;
        if (tc_shape(M, N, K, bits, G_of_plan, dtype, w16, &ts)) {
            pl->maxm = maxm; pl->R = 1; pl->wide = 1; pl->tc = 1; pl->npass = ts.npass;
            pl->wk = ts.wk; pl->wr = ts.wr; pl->tile_iters = ts.tsb; pl->C = ts.sb; pl->smem = ts.smem;
            pl->grid = dim3((unsigned)ts.gx, 1, (unsigned)batch);
            pl->block = dim3(32 * ts.wk * ts.wr, 1, 1);
            return QMV_OK;
        }
    }

    if (g_forced.path == 1 && w16 && (K % c_wide == 0)) wide = true;
    const int U = wide ? fi.wide_units : 1;
    const int C = 32 * U;
    const int NC = K / C;
    const int sms = device_sms();

    int R = 1, wk = 1, wr = 1;
    if (N <= 64) {
        // narrow N: one row per warp, the row's chunks spread over the block
        R = 1;
        wr = 1;
        wk = (NC + 31) / 32;
        wk = wk < 1 ? 1 : (wk > 8 ? 8 : wk);
        if (N * wk < 2 * sms && NC >= 64 * wk) {  // still few threads: more warps per row
            while (wk < 8 && NC >= 32 * (wk + 1)) ++wk;
        }
    } else {
        const int rcap = wide ? rows_per_warp_cap(fi.bits, maxm) : 1;
        R = N >= 1024 ? rcap : (N >= 256 ? (rcap < 2 ? rcap : 2) : 1);
        const long long warps = ((long long)N + R - 1) / R * batch;
        // k-warps: at least 2 for long rows (>= 256 chunks: more loads in
        // flight per row; not for 6-bit, whose 12-word chunks already fill
        // the registers), more while the GPU holds fewer than ~8 warps per SM
        // (the block-scaled and signed-int families: one k-warp and 8 row
        // warps, measured best on B200 for 4- and 8-bit codes at 16384^2)
        wk = (aff && NC >= 256 && fi.bits != 6) ? 2 : 1;
        while (wk < 8 && warps * wk < (long long)sms * 8 && NC >= 64 * wk) wk *= 2;
        wr = wk >= 8 ? 1 : 8 / wk;
        if (aff && wr > 4 && wk == 1) wr = 4;
    }
    if (g_forced.R > 0) R = g_forced.R;
    if (g_forced.wk > 0) wk = g_forced.wk;
    if (g_forced.wr > 0) wr = g_forced.wr;
    if (pair) {
        if (R < 2) R = 2;
        if (!qmv::pair_shape_instantiated(maxm, R, wide)) R = 2;
    } else if (qkv) {
        if (!qmv::qkv_shape_instantiated(maxm, R, wide)) R = wide ? (maxm <= 2 ? 4 : 2) : 1;
    } else if (!qmv::shape_instantiated(maxm, R, wide)) {
        R = 1;
    }
    if (wk < 1) wk = 1;
    if (wk > 8) wk = 8;
    if (wr < 1) wr = 1;
    while (wk * wr > 8) --wr;
    if (wr < 1) wr = 1;

    // x tile: shrink the k-warps until one iteration of x fits the budget
    const size_t budget = 96 * 1024;
    auto per_iter_of = [&](int wk_) {
        return (size_t)maxm * C * 32 * wk_ * 4 + (affl ? (size_t)maxm * U * 32 * wk_ * 4 : 0);
    };
    while (wk > 1 && per_iter_of(wk) > budget) --wk;
    const int KT = 32 * wk;
    const size_t per_iter = per_iter_of(wk);
    const size_t red = (size_t)wk * wr * R * maxm * 4;
    long long iters_needed = ((long long)NC + KT - 1) / KT;
    if (iters_needed < 1) iters_needed = 1;
    long long ti = (long long)((budget > red ? budget - red : 0) / per_iter);
    if (ti < 1) ti = 1;
    if (ti > iters_needed) ti = iters_needed;
    const size_t smem = per_iter * ti + red + (norm ? 512 : 0);     // + the RMSNorm partial sums
    if (smem > (size_t)qmv::kMaxSmem) return QMV_EUNSUPPORTED;

    const long long rows_per_block = (long long)wr * R;
    const long long gx = ((long long)N + rows_per_block - 1) / rows_per_block;
    if (gx > 0x7FFFFFFFLL) return QMV_EINVAL;

    pl->maxm = maxm; pl->R = R; pl->wide = wide; pl->tc = 0; pl->npass = 0; pl->wk = wk; pl->wr = wr;
    pl->tile_iters = (int)ti; pl->C = C; pl->smem = smem;
    pl->grid = dim3((unsigned)gx, 1, (unsigned)batch);
    pl->block = dim3(32 * wk * wr, 1, 1);
    return QMV_OK;
}

int finish(cudaError_t e) {
    if (e == cudaSuccess) return QMV_OK;
    g_last_cuda = (int)e;
    cudaGetLastError();  // clear the sticky-free launch error state
    return QMV_ECUDA;
}

bool pdl_enabled() {
    static int v = -1;
    if (v < 0) {
        const char* s = getenv("QMV_PDL");
        v = (s && s[0] == '0') ? 0 : 1;
    }
    return v == 1;
}

int check_common(const void* x, const void* w, const void* s, void* y, int M, int N, int K, int dtype) {
    if (M < 0 || N < 0 || K < 0) return QMV_EINVAL;
    if (M > QMV_MAX_M) return QMV_EUNSUPPORTED;
    if (dtype != QMV_F32 && dtype != QMV_F16 && dtype != QMV_BF16) return QMV_EUNSUPPORTED;
    if (M == 0 || N == 0) return QMV_OK;
    if (!y || (K > 0 && (!x || !w || !s))) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (!aligned(y, eb) || (x && !aligned(x, eb))) return QMV_EALIGN;
    if (w && !aligned(w, 4)) return QMV_EALIGN;
    return QMV_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

// [batch][N][row bytes / 8] packed rows as a 3-D tensor map of 8-byte
// elements with box {box0, rows, 1}; out-of-range elements read as zero.
bool encode_rows_map(CUtensorMap* m, const void* base, long long row_bytes, int N, int batch, int box0, int rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)(row_bytes / 8), (cuuint64_t)N, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * (cuuint64_t)N};
    const cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// As encode_rows_map with the 128-byte swizzle (box {16, rows, 1}: 128 bytes
// a row), for the tensor-memory kernel's conflict-free row reads.
bool encode_rows_map_sw128(CUtensorMap* m, const void* base, long long row_bytes, int N, int batch, int rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)(row_bytes / 8), (cuuint64_t)N, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * (cuuint64_t)N};
    const cuuint32_t box[3] = {16, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [batch][N][K/G] scales (or biases) as a 3-D tensor map with box
// {box0 groups, rows, 1}; out-of-range elements read as zero.
bool encode_scale_map(CUtensorMap* m, const void* base, int dtype, long long KG, int N, int batch, int box0,
                      int rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const CUtensorMapDataType dt = dtype == QMV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : dtype == QMV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t es = (cuuint64_t)elem_bytes(dtype);
    const cuuint64_t dims[3] = {(cuuint64_t)KG, (cuuint64_t)N, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)KG * es, (cuuint64_t)KG * es * (cuuint64_t)N};
    const cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// The same for block scales of 1, 2 or 4 bytes (the FP formats' E8M0 / E4M3
// bytes, FP16 or FP32), copied as raw elements.
bool encode_scale_map_es(CUtensorMap* m, const void* base, int es, long long KG, int N, int batch, int box0, int rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const CUtensorMapDataType dt = es == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32
                                 : es == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                           : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const cuuint64_t dims[3] = {(cuuint64_t)KG, (cuuint64_t)N, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)KG * es, (cuuint64_t)KG * es * (cuuint64_t)N};
    const cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Bytes of one block scale of an FP family (skind for the run-time-scaled ones).
int fp_scale_bytes(int fam, int skind) {
    if (fam == qmv::FAM_E2M1 || fam == qmv::FAM_E4M3 || fam == qmv::FAM_E5M2 || fam == qmv::FAM_SINT)
        return skind == qmv::SK_F32 ? 4 : skind == qmv::SK_F16 ? 2 : 1;
    return 1;
}

int run(int fam, const void* x, const void* w, const void* scales, const void* biases,
        const float* gscale, void* y, int M, int N, int K, int bits, int G, int dtype, int batch,
        int x_batched, void* stream, const int* ids = nullptr, int n_experts = 0, bool qmm = false,
        int skind = 0) {
    const long long row_bytes = (long long)K * fmt_info(fam, bits).bits / 8;
    Plan pl;
    const bool w16 = aligned(w, 16);
    const bool aff = fam == qmv::FAM_AFFINE;
    const bool s16 = aligned(scales, 16) && (!aff || aligned(biases, 16));
    const bool x16 = aligned(x, 16) && ((size_t)K * elem_bytes(dtype)) % 16 == 0;
    const int fes = fp_scale_bytes(fam, skind);
    int st = make_plan(fam, M, N, K, bits, G, dtype, w16, batch, &pl, s16, ids != nullptr, false, x16, qmm, false,
                       false, fes);
    if (st != QMV_OK) return st;
    // M > 8 (qmm): only the tensor-memory kernel and the tensor-core ring take it
    if (M > QMV_MAX_M && pl.tc != 5 && pl.tc != 2 && pl.tc != 6) return QMV_EUNSUPPORTED;
    qmv::Params p{};
    if (pl.tc == 5) {
        // tensor-memory kernel: swizzled row boxes, scale / bias boxes of 8 groups
        if (!encode_rows_map_sw128(&p.wmap, w, row_bytes, N, batch, 128) ||
            !encode_scale_map(&p.smap, scales, dtype, K / G, N, batch, 8, 128) ||
            !encode_scale_map(&p.bmap, biases, dtype, K / G, N, batch, 8, 128)) {
            cudaGetLastError();
            return QMV_ECUDA;
        }
    }
    if (pl.tc == 6) {
        // per-group ring: swizzled 128-byte row boxes, scale / bias tiles of 8 groups
        const int rows = 16 * pl.wr;
        if (!encode_rows_map_sw128(&p.wmap, w, row_bytes, N, batch, rows) ||
            !encode_scale_map(&p.smap, scales, dtype, K / G, N, batch, 8, rows) ||
            !encode_scale_map(&p.bmap, biases, dtype, K / G, N, batch, 8, rows)) {
            cudaGetLastError();
            return QMV_ECUDA;
        }
    }
    const bool ring = pl.tc == 2 || pl.tc == 4;        // the weight-ring kernels
    if (ring && pl.sring) {
        const int rows = 16 * pl.wr;
        bool okm;
        if (aff) {
            const int box0 = pl.sbw / elem_bytes(dtype);
            okm = encode_scale_map(&p.smap, scales, dtype, K / G, N, batch, box0, rows) &&
                  encode_scale_map(&p.bmap, biases, dtype, K / G, N, batch, box0, rows);
        } else {
            okm = encode_scale_map_es(&p.smap, scales, fes, K / G, N, batch, pl.sbw / fes, rows);
        }
        if (!okm) {
            cudaGetLastError();
            st = make_plan(fam, M, N, K, bits, G, dtype, w16, batch, &pl, false, false, false, x16, qmm, false, false,
                           fes);                                          // scales from global memory
            if (st != QMV_OK) return st;
        }
    }
    // the packed rows' tensor map, for the final plan
    if (ring && !encode_rows_map(&p.wmap, w, row_bytes, N, batch, pl.pitch / 8, 16 * pl.wr)) {
        cudaGetLastError();
        return QMV_ECUDA;
    }
    p.x = x; p.w = static_cast<const uint8_t*>(w); p.scales = scales; p.biases = biases;
    p.gscale = gscale; p.y = y;
    p.M = M; p.N = N; p.K = K; p.G = G;
    p.wk = pl.wk; p.wr = pl.wr; p.tile_iters = pl.tile_iters;
    const size_t eb = elem_bytes(dtype);
    p.x_vec = (aligned(x, 16) && ((size_t)K * eb) % 16 == 0) ? 1 : 0;
    p.x_bs = x_batched ? (long long)M * K : 0;
    p.w_bs = (long long)N * row_bytes;
    p.s_bs = (long long)N * (K / G);
    p.y_bs = (long long)M * N;
    p.w_row = row_bytes;
    // gather reads ids (often written by the kernel just before) ahead of its
    // grid-dependency wait: it launches without programmatic dependent launch
    qmv::Launch L{pl.grid, pl.block, pl.smem, static_cast<cudaStream_t>(stream), pdl_enabled() && !ids};
    p.ids = ids;
    p.n_experts = n_experts;
    p.gamma = nullptr; p.eps = 0.f;
    p.skind = skind;
    p.test_skip = g_test_skip.load(std::memory_order_relaxed);
    cudaError_t e;
    p.sps = pl.sps; p.pitch = pl.pitch; p.fault = nullptr;
    p.sring = pl.sring; p.soff = pl.soff; p.boff = pl.boff; p.sbw = pl.sbw;
    p.kf32 = 0x4B000000u;
    p.kbf16 = 0x43004300u;
    if (pl.tc == 6) {
        p.fault = fault_word();
        if (!p.fault) return QMV_ECUDA;
        return finish(qmv::launch_tcg_affine(dtype, G, pl.npass, p, L));
    }
    if (pl.tc == 2) {
        p.fault = fault_word();
        if (!p.fault) return QMV_ECUDA;
        return finish(qmv::launch_tcb_affine(bits, dtype, pl.npass, pl.spb, pl.wk * pl.wr, p, L));
    }
    if (pl.tc == 4) {
        p.fault = fault_word();
        if (!p.fault) return QMV_ECUDA;
        return finish(fam == qmv::FAM_AFFINE ? qmv::launch_tcf_affine(bits, pl.wk * pl.wr, p, L)
                                             : qmv::launch_tcf_fp(fam, pl.wk * pl.wr, p, L));
    }
    if (pl.tc == 5) {
        p.fault = fault_word();
        if (!p.fault) return QMV_ECUDA;
        return finish(qmv::launch_umma_affine(bits, pl.mld, p, pl.um, L));
    }
    if (pl.tc == 3) return finish(qmv::launch_direct(fam, bits, dtype, pl.maxm, pl.wide != 0, p, L));
    if (pl.tc) return finish(qmv::launch_tc_affine(bits, dtype, pl.npass, p, L));
    if (fam == qmv::FAM_AFFINE) {
        switch (bits) {
            case 2: e = qmv::launch_affine_b2(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
            case 3: e = qmv::launch_affine_b3(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
            case 4: e = qmv::launch_affine_b4(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
            case 5: e = qmv::launch_affine_b5(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
            case 6: e = qmv::launch_affine_b6(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
            case 8: e = qmv::launch_affine_b8(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
            default: return QMV_EUNSUPPORTED;
        }
    } else if (fam == qmv::FAM_SINT) {
        e = qmv::launch_sint(bits, dtype, pl.maxm, pl.R, pl.wide, p, L);
    } else {
        e = qmv::launch_fp(fam, dtype, pl.maxm, pl.R, pl.wide, p, L);
    }
    return finish(e);
}

// The fused gate + up projection with SwiGLU: the row-tiled CUDA-core kernel
// over the 2N interleaved rows of the pair.
int run_pair(const void* x, const void* wg, const void* sg, const void* bg, const void* wu, const void* su,
             const void* bu, const float* route_w, void* y, int M, int N, int K, int bits, int G, int dtype,
             float clamp, void* stream) {
    const long long row_bytes = (long long)K * bits / 8;
    Plan pl;
    const bool w16 = aligned(wg, 16) && aligned(wu, 16);
    int st = make_plan(qmv::FAM_AFFINE, M, 2 * N, K, bits, G, dtype, w16, 1, &pl, false, true, true);
    if (st != QMV_OK) return st;
    if (pl.tc != 0) return QMV_EUNSUPPORTED;       // the row-tiled kernel's launch shape only
    qmv::Params p{};
    p.x = x; p.w = static_cast<const uint8_t*>(wg); p.scales = sg; p.biases = bg; p.gscale = nullptr; p.y = y;
    p.w2 = static_cast<const uint8_t*>(wu); p.scales2 = su; p.biases2 = bu;
    p.route_w = route_w; p.act_clamp = clamp;
    p.gamma = nullptr; p.eps = 0.f;
    p.M = M; p.N = N; p.K = K; p.G = G;
    p.wk = pl.wk; p.wr = pl.wr; p.tile_iters = pl.tile_iters;
    const size_t eb = elem_bytes(dtype);
    p.x_vec = (aligned(x, 16) && ((size_t)K * eb) % 16 == 0) ? 1 : 0;
    p.x_bs = 0; p.w_bs = 0; p.s_bs = 0; p.y_bs = 0;
    p.w_row = row_bytes;
    p.ids = nullptr; p.n_experts = 0;
    p.sps = 0; p.pitch = 0; p.fault = nullptr; p.sring = 0; p.soff = 0; p.boff = 0; p.sbw = 0;
    p.kf32 = 0x4B000000u;
    p.kbf16 = 0x43004300u;
    qmv::Launch L{pl.grid, pl.block, pl.smem, static_cast<cudaStream_t>(stream), pdl_enabled()};
    return finish(qmv::launch_affine_pair(bits, dtype, pl.maxm, pl.R, pl.wide != 0, p, L));
}

// qmm beyond QMV_MAX_M rows: the tensor-memory kernel (one launch, each
// weight decoded once) where the matrix has few 128-row tiles -- its K split
// over a cluster keeps the SMs busy; measured on B200 (4-bit g64 bf16, M 16 /
// 32 / 64): 4096 x 4096 27.6 / 37.2 / 101 us against 38.6 / 72.0 / 139 us in
// 16-row chunks, 4096 x 14336 67 / 127 us against 104 / 199 us; for 28672 x
// 4096 the chunks win (96 / 189 / 375 against 140 / 274 / 473 us).
bool qmm_prefers_umma(int M, int N, int K, int bits, int G, int dtype, bool w16, bool s16) {
    if (g_forced.path == 7) return true;
    if (g_forced.path >= 0 || N > 5120) return false;
    TcgShape tg;      // the per-group tensor-core ring, where it applies, measured faster
    return !(tcg_preferred(M > 32 ? 32 : M, N, bits) && tcg_shape(M > 32 ? 32 : M, N, K, bits, G, dtype, w16, s16, &tg));
}

// x rows per launch of qmv_qmm_affine beyond QMV_MAX_M rows: 32 or 16 when
// the tensor-core ring kernel takes that many (x rows x groups of a
// super-block <= 32 slot columns; more than 64 output rows), else QMV_MAX_M.
int qmm_chunk(int M, int N, int K, int bits, int G, int dtype, bool w16, bool s16) {
    if (M <= QMV_MAX_M || N <= 64 || K <= 0) return QMV_MAX_M;
    // the per-group tensor-core ring takes up to 32 rows a launch
    const int c0 = M > 16 ? 32 : 16;
    if (g_forced.path == 8 || (g_forced.path < 0 && tcg_preferred(c0, N, bits))) {
        TcgShape tg;
        if (tcg_shape(c0, N, K, bits, G, dtype, w16, s16, &tg)) return c0;
    }
    for (int c : {32, 16}) {
        if (c >= M + QMV_MAX_M) continue;
        TcbShape ts;
        if (tcb_shape(c, N, K, bits, G, dtype, w16, s16, &ts)) return c;
    }
    return QMV_MAX_M;
}

// Fills the Params fields every row-tiled launch takes.
void base_params(qmv::Params* p, const Plan& pl, const void* x, const void* w, const void* s, const void* b, void* y,
                 int M, int N, int K, int bits, int G, int dtype) {
    p->x = x; p->w = static_cast<const uint8_t*>(w); p->scales = s; p->biases = b; p->gscale = nullptr; p->y = y;
    p->M = M; p->N = N; p->K = K; p->G = G;
    p->wk = pl.wk; p->wr = pl.wr; p->tile_iters = pl.tile_iters;
    const size_t eb = elem_bytes(dtype);
    p->x_vec = (aligned(x, 16) && ((size_t)K * eb) % 16 == 0) ? 1 : 0;
    p->x_bs = 0; p->w_bs = 0; p->s_bs = 0; p->y_bs = 0;
    p->w_row = (long long)K * bits / 8;
    p->ids = nullptr; p->n_experts = 0;
    p->sps = 0; p->pitch = 0; p->fault = nullptr; p->sring = 0; p->soff = 0; p->boff = 0; p->sbw = 0;
    p->kf32 = 0x4B000000u;
    p->kbf16 = 0x43004300u;
}

// Q / K / V in one call: the row-tiled CUDA-core kernel over the Nq + 2 Nkv
// output rows, each row reading its own matrix.
int run_qkv(const void* x, const void* const (&w)[3], const void* const (&s)[3], const void* const (&b)[3], void* y,
            int M, int Nq, int Nkv, int K, int bits, int G, int dtype, void* stream) {
    const int N = Nq + 2 * Nkv;
    Plan pl;
    const bool w16 = aligned(w[0], 16) && aligned(w[1], 16) && aligned(w[2], 16);
    int st = make_plan(qmv::FAM_AFFINE, M, N, K, bits, G, dtype, w16, 1, &pl, false, true, false, true, false, true);
    if (st != QMV_OK) return st;
    if (pl.tc != 0) return QMV_EUNSUPPORTED;       // the row-tiled kernel's launch shape only
    qmv::Params p{};
    base_params(&p, pl, x, w[0], s[0], b[0], y, M, N, K, bits, G, dtype);
    p.w2 = static_cast<const uint8_t*>(w[1]); p.scales2 = s[1]; p.biases2 = b[1];
    p.w3 = static_cast<const uint8_t*>(w[2]); p.scales3 = s[2]; p.biases3 = b[2];
    p.n1 = Nq; p.n2 = Nq + Nkv;
    qmv::Launch L{pl.grid, pl.block, pl.smem, static_cast<cudaStream_t>(stream), pdl_enabled()};
    return finish(qmv::launch_affine_qkv(bits, dtype, pl.maxm, pl.R, pl.wide != 0, p, L));
}

// RMSNorm fused into the row-tiled CUDA-core kernel's x staging.
int run_rms_norm(const void* x, const void* gamma, float eps, const void* w, const void* s, const void* b, void* y,
                 int M, int N, int K, int bits, int G, int dtype, void* stream) {
    Plan pl;
    int st = make_plan(qmv::FAM_AFFINE, M, N, K, bits, G, dtype, aligned(w, 16), 1, &pl, false, true, false, true,
                       false, false, true);
    if (st != QMV_OK) return st;
    if (pl.tc != 0) return QMV_EUNSUPPORTED;       // the row-tiled kernel's launch shape only
    qmv::Params p{};
    base_params(&p, pl, x, w, s, b, y, M, N, K, bits, G, dtype);
    p.gamma = gamma; p.eps = eps;
    qmv::Launch L{pl.grid, pl.block, pl.smem, static_cast<cudaStream_t>(stream), pdl_enabled()};
    cudaError_t e;
    switch (bits) {
        case 2: e = qmv::launch_affine_b2(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
        case 3: e = qmv::launch_affine_b3(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
        case 4: e = qmv::launch_affine_b4(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
        case 5: e = qmv::launch_affine_b5(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
        case 6: e = qmv::launch_affine_b6(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
        case 8: e = qmv::launch_affine_b8(dtype, pl.maxm, pl.R, pl.wide, p, L); break;
        default: return QMV_EUNSUPPORTED;
    }
    return finish(e);
}

int check_affine(int bits, int group) {
    if (bits != 2 && bits != 3 && bits != 4 && bits != 5 && bits != 6 && bits != 8) return QMV_EUNSUPPORTED;
    if (group != 32 && group != 64 && group != 128) return QMV_EUNSUPPORTED;
    return QMV_OK;
}

int fp_family(int mode) {
    return mode == QMV_MXFP4 ? qmv::FAM_MXFP4 : mode == QMV_NVFP4 ? qmv::FAM_NVFP4
         : mode == QMV_MXFP8_E4M3 ? qmv::FAM_MXFP8 : -1;
}

int check_fp(int mode, int K, const float* gscale) {
    int fam = fp_family(mode);
    if (fam < 0) return QMV_EUNSUPPORTED;
    if (mode == QMV_NVFP4) {
        if (K % 16 != 0) return QMV_EINVAL;
        if (!gscale) return QMV_EINVAL;
        if (!aligned(gscale, 4)) return QMV_EALIGN;
    } else {
        if (K % 32 != 0) return QMV_EINVAL;
        if (gscale) return QMV_EINVAL;
    }
    return QMV_OK;
}

// The Track-1 formats (qmv_format): kernel family, bits per code, block,
// scale type, global scale.  The three formats of qmv_fp keep their own
// families; the rest run on the run-time-scaled E2M1 / E4M3 / E5M2 families
// or on the signed-integer family.
struct BsFmt {
    int fam, bits, block, skind, global;
};
constexpr int kSF32 = qmv::SK_F32, kSF16 = qmv::SK_F16, kSE8 = qmv::SK_E8M0, kSE4 = qmv::SK_E4M3;
const BsFmt kBsFmt[QMV_FMT_COUNT] = {
    {qmv::FAM_NVFP4, 4, 16, kSE4, 1}, {qmv::FAM_MXFP4, 4, 32, kSE8, 0},
    {qmv::FAM_MXFP8, 8, 32, kSE8, 0}, {qmv::FAM_E5M2, 8, 32, kSE8, 0},
    {qmv::FAM_E4M3, 8, 16, kSF32, 0}, {qmv::FAM_E2M1, 4, 32, kSF32, 0},
    {qmv::FAM_E4M3, 8, 32, kSF32, 0}, {qmv::FAM_E5M2, 8, 32, kSF32, 0},
    {qmv::FAM_SINT, 2, 64, kSF32, 0}, {qmv::FAM_SINT, 3, 64, kSF32, 0}, {qmv::FAM_SINT, 4, 64, kSF32, 0},
    {qmv::FAM_SINT, 5, 64, kSF32, 0}, {qmv::FAM_SINT, 6, 64, kSF32, 0}, {qmv::FAM_SINT, 8, 64, kSF32, 0},
    {qmv::FAM_SINT, 2, 32, kSE8, 0}, {qmv::FAM_SINT, 3, 32, kSE8, 0}, {qmv::FAM_SINT, 4, 32, kSE8, 0},
    {qmv::FAM_SINT, 5, 32, kSE8, 0}, {qmv::FAM_SINT, 6, 32, kSE8, 0}, {qmv::FAM_SINT, 8, 32, kSE8, 0},
    {qmv::FAM_E4M3, 8, 16, kSF16, 0}, {qmv::FAM_E2M1, 4, 32, kSF16, 0},
    {qmv::FAM_E4M3, 8, 32, kSF16, 0}, {qmv::FAM_E5M2, 8, 32, kSF16, 0},
    {qmv::FAM_SINT, 2, 64, kSF16, 0}, {qmv::FAM_SINT, 3, 64, kSF16, 0}, {qmv::FAM_SINT, 4, 64, kSF16, 0},
    {qmv::FAM_SINT, 5, 64, kSF16, 0}, {qmv::FAM_SINT, 6, 64, kSF16, 0}, {qmv::FAM_SINT, 8, 64, kSF16, 0},
};

int scale_bytes_of(int skind) { return skind == qmv::SK_F32 ? 4 : skind == qmv::SK_F16 ? 2 : 1; }

// Argument checks shared by the block-scaled entries (format, K, global, scales).
int check_bs(int format, int K, const void* scales, const float* gscale, const BsFmt** out) {
    if (format < 0 || format >= QMV_FMT_COUNT) return QMV_EUNSUPPORTED;
    const BsFmt& f = kBsFmt[format];
    if (K % f.block != 0) return QMV_EINVAL;
    if (f.global) {
        if (!gscale) return QMV_EINVAL;
        if (!aligned(gscale, 4)) return QMV_EALIGN;
    } else if (gscale) {
        return QMV_EINVAL;
    }
    if (scales && !aligned(scales, scale_bytes_of(f.skind))) return QMV_EALIGN;
    *out = &f;
    return QMV_OK;
}

}  // namespace

extern "C" {

int qmv_affine_batched(const void* x, const void* w_packed, const void* scales, const void* biases,
                       void* y, int M, int N, int K, int bits, int group_size, int dtype, int batch,
                       int x_batched, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (batch < 1 || batch > 65535 || (x_batched != 0 && x_batched != 1)) return QMV_EINVAL;
    if (K % group_size != 0) return QMV_EINVAL;
    st = check_common(x, w_packed, scales, y, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    if (K > 0 && !biases) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (K > 0 && (!aligned(scales, eb) || !aligned(biases, eb))) return QMV_EALIGN;
    return run(qmv::FAM_AFFINE, x, w_packed, scales, biases, nullptr, y, M, N, K, bits, group_size,
               dtype, batch, x_batched, stream);
}

int qmv_affine(const void* x, const void* w_packed, const void* scales, const void* biases, void* y,
               int M, int N, int K, int bits, int group_size, int dtype, void* stream) {
    return qmv_affine_batched(x, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, 1, 1,
                              stream);
}

int qmv_fp_batched(const void* x, const void* w_packed, const void* scales, const float* global_scale,
                   void* y, int M, int N, int K, int mode, int dtype, int batch, int x_batched,
                   void* stream) {
    int st = check_fp(mode, K, global_scale);
    if (st != QMV_OK) return st;
    if (batch < 1 || batch > 65535 || (x_batched != 0 && x_batched != 1)) return QMV_EINVAL;
    st = check_common(x, w_packed, scales, y, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    const int fam = fp_family(mode);
    const int G = mode == QMV_NVFP4 ? 16 : 32;
    return run(fam, x, w_packed, scales, nullptr, global_scale, y, M, N, K, 0, G, dtype, batch,
               x_batched, stream);
}

int qmv_fp(const void* x, const void* w_packed, const void* scales, const float* global_scale, void* y,
           int M, int N, int K, int mode, int dtype, void* stream) {
    return qmv_fp_batched(x, w_packed, scales, global_scale, y, M, N, K, mode, dtype, 1, 1, stream);
}

int qmv_block_scaled_batched(const void* x, const void* w_packed, const void* scales, const float* global_scale,
                             void* y, int M, int N, int K, int format, int dtype, int batch, int x_batched,
                             void* stream) {
    const BsFmt* f = nullptr;
    int st = check_bs(format, K, scales, global_scale, &f);
    if (st != QMV_OK) return st;
    if (batch < 1 || batch > 65535 || (x_batched != 0 && x_batched != 1)) return QMV_EINVAL;
    st = check_common(x, w_packed, scales, y, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    return run(f->fam, x, w_packed, scales, nullptr, global_scale, y, M, N, K, f->bits, f->block, dtype, batch,
               x_batched, stream, nullptr, 0, false, f->skind);
}

int qmv_block_scaled(const void* x, const void* w_packed, const void* scales, const float* global_scale, void* y,
                     int M, int N, int K, int format, int dtype, void* stream) {
    return qmv_block_scaled_batched(x, w_packed, scales, global_scale, y, M, N, K, format, dtype, 1, 1, stream);
}

int qmv_dequant_block_scaled_f32(const void* w_packed, const void* scales, const float* global_scale,
                                 float* w_out, int N, int K, int format, void* stream) {
    const BsFmt* f = nullptr;
    int st = check_bs(format, K, scales, global_scale, &f);
    if (st != QMV_OK) return st;
    if (N < 0 || K < 0) return QMV_EINVAL;
    if (N == 0 || K == 0) return QMV_OK;
    if (!w_packed || !scales || !w_out) return QMV_EINVAL;
    if (!aligned(w_packed, 4) || !aligned(w_out, 16)) return QMV_EALIGN;
    return finish(qmv::launch_dequant(f->fam, f->bits, 0, static_cast<const uint8_t*>(w_packed), scales, nullptr,
                                      global_scale, w_out, N, K, f->block, (long long)K * f->bits / 8,
                                      static_cast<cudaStream_t>(stream), f->skind));
}

int qmv_format_info(int format, int* element_bits, int* block, int* scale_bytes, int* has_global) {
    if (format < 0 || format >= QMV_FMT_COUNT) return QMV_EUNSUPPORTED;
    const BsFmt& f = kBsFmt[format];
    if (element_bits) *element_bits = f.bits;
    if (block) *block = f.block;
    if (scale_bytes) *scale_bytes = scale_bytes_of(f.skind);
    if (has_global) *has_global = f.global;
    return QMV_OK;
}

int qmv_dequant_affine_f32(const void* w_packed, const void* scales, const void* biases, float* w_out,
                           int N, int K, int bits, int group_size, int dtype, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (dtype != QMV_F32 && dtype != QMV_F16 && dtype != QMV_BF16) return QMV_EUNSUPPORTED;
    if (N < 0 || K < 0 || K % group_size != 0) return QMV_EINVAL;
    if (N == 0 || K == 0) return QMV_OK;
    if (!w_packed || !scales || !biases || !w_out) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (!aligned(w_packed, 4) || !aligned(scales, eb) || !aligned(biases, eb) || !aligned(w_out, 16))
        return QMV_EALIGN;
    return finish(qmv::launch_dequant(qmv::FAM_AFFINE, bits, dtype, static_cast<const uint8_t*>(w_packed),
                                      scales, biases, nullptr, w_out, N, K, group_size,
                                      (long long)K * bits / 8, static_cast<cudaStream_t>(stream)));
}

int qmv_dequant_fp_f32(const void* w_packed, const void* scales, const float* global_scale, float* w_out,
                       int N, int K, int mode, void* stream) {
    int st = check_fp(mode, K, global_scale);
    if (st != QMV_OK) return st;
    if (N < 0 || K < 0) return QMV_EINVAL;
    if (N == 0 || K == 0) return QMV_OK;
    if (!w_packed || !scales || !w_out) return QMV_EINVAL;
    if (!aligned(w_packed, 4) || !aligned(w_out, 16)) return QMV_EALIGN;
    const int fam = fp_family(mode);
    const int bits = fam == qmv::FAM_MXFP8 ? 8 : 4;
    return finish(qmv::launch_dequant(fam, bits, 0, static_cast<const uint8_t*>(w_packed), scales, nullptr,
                                      global_scale, w_out, N, K, mode == QMV_NVFP4 ? 16 : 32,
                                      (long long)K * bits / 8, static_cast<cudaStream_t>(stream)));
}

int qmv_quantize_affine(const void* w, void* w_packed, void* scales, void* biases, int N, int K, int bits,
                        int group_size, int dtype, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (dtype != QMV_F32 && dtype != QMV_F16 && dtype != QMV_BF16) return QMV_EUNSUPPORTED;
    if (N < 0 || K < 0 || K % group_size != 0) return QMV_EINVAL;
    if (N == 0 || K == 0) return QMV_OK;
    if (!w || !w_packed || !scales || !biases) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (!aligned(w, eb) || !aligned(w_packed, 4) || !aligned(scales, eb) || !aligned(biases, eb)) return QMV_EALIGN;
    // 2: coalesced tiles (w and w_packed 16-byte aligned); 1: 16-byte loads of
    // w per thread; 0: element loads
    const int vec = (aligned(w, 16) && ((size_t)K * eb) % 16 == 0) ? (aligned(w_packed, 16) ? 2 : 1) : 0;
    return finish(qmv::launch_quantize_affine(bits, dtype, w, w_packed, scales, biases, N, K, group_size, vec,
                                              static_cast<cudaStream_t>(stream)));
}

int qmv_quantize_fp(const void* w, void* w_packed, void* scales, const float* global_scale, int N, int K,
                    int mode, int dtype, void* stream) {
    if (fp_family(mode) < 0) return QMV_EUNSUPPORTED;
    if (dtype != QMV_F32 && dtype != QMV_F16 && dtype != QMV_BF16) return QMV_EUNSUPPORTED;
    const int blk = mode == QMV_NVFP4 ? 16 : 32;
    if (N < 0 || K < 0 || K % blk != 0) return QMV_EINVAL;
    if ((mode == QMV_NVFP4) != (global_scale != nullptr)) return QMV_EINVAL;
    if (N == 0 || K == 0) return QMV_OK;
    if (!w || !w_packed || !scales) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (!aligned(w, eb) || (global_scale && !aligned(global_scale, 4))) return QMV_EALIGN;
    const bool vec = aligned(w, 16) && aligned(w_packed, mode == QMV_NVFP4 ? 8 : 16);
    return finish(qmv::launch_quantize_fp(mode, dtype, w, w_packed, scales, global_scale, N, K, vec,
                                          static_cast<cudaStream_t>(stream)));
}

int qmv_affine_gather(const void* x, const void* w_packed, const void* scales, const void* biases,
                      const int* expert_ids, void* y, int M, int N, int K, int bits, int group_size, int dtype,
                      int n_tokens, int n_experts, int x_batched, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (n_tokens < 1 || n_tokens > 65535 || n_experts < 1 || (x_batched != 0 && x_batched != 1))
        return QMV_EINVAL;
    if (K % group_size != 0) return QMV_EINVAL;
    st = check_common(x, w_packed, scales, y, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    if (!expert_ids || (K > 0 && !biases)) return QMV_EINVAL;
    if (!aligned(expert_ids, 4)) return QMV_EALIGN;
    const size_t eb = elem_bytes(dtype);
    if (K > 0 && (!aligned(scales, eb) || !aligned(biases, eb))) return QMV_EALIGN;
    return run(qmv::FAM_AFFINE, x, w_packed, scales, biases, nullptr, y, M, N, K, bits, group_size, dtype, n_tokens,
               x_batched, stream, expert_ids, n_experts);
}

int qmv_qmm_affine(const void* x, const void* w_packed, const void* scales, const void* biases, void* y,
                   int M, int N, int K, int bits, int group_size, int dtype, void* stream) {
    if (M < 0 || M > QMV_QMM_MAX_M) return QMV_EINVAL;
    // every argument is checked once, on the first chunk: the later chunks
    // differ only by whole-row offsets of x and y, which keep the alignment
    const int m1 = M < QMV_MAX_M ? M : QMV_MAX_M;
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (K % group_size != 0) return QMV_EINVAL;
    st = check_common(x, w_packed, scales, y, m1, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    if (K > 0 && !biases) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (K > 0 && (!aligned(scales, eb) || !aligned(biases, eb))) return QMV_EALIGN;
    // more than QMV_MAX_M rows: the tensor-memory kernel takes them all in one
    // launch for matrices of few row tiles (qmm_prefers_umma, when its layout
    // rules hold); otherwise the tensor-core ring kernel takes up to 32 rows a
    // launch (its 32 slot columns: x rows x groups of a super-block), and the
    // rest go in chunks of QMV_MAX_M
    int chunk = QMV_MAX_M;
    if (M > QMV_MAX_M) {
        if (qmm_prefers_umma(M, N, K, bits, group_size, dtype, aligned(w_packed, 16),
                             aligned(scales, 16) && aligned(biases, 16))) {
            st = run(qmv::FAM_AFFINE, x, w_packed, scales, biases, nullptr, y, M, N, K, bits, group_size, dtype, 1, 1,
                     stream, nullptr, 0, true);
            if (st != QMV_EUNSUPPORTED) return st;
        }
        chunk = qmm_chunk(M, N, K, bits, group_size, dtype, aligned(w_packed, 16),
                          aligned(scales, 16) && aligned(biases, 16));
    }
    // chunks, back to back on the stream: a weight matrix that fits in L2 is
    // read from HBM by the first chunk only
    for (int m0 = 0; m0 < M; m0 += chunk) {
        const int mc = M - m0 < chunk ? M - m0 : chunk;
        const void* xc = x ? static_cast<const char*>(x) + (size_t)m0 * K * eb : nullptr;
        void* yc = static_cast<char*>(y) + (size_t)m0 * N * eb;
        st = run(qmv::FAM_AFFINE, xc, w_packed, scales, biases, nullptr, yc, mc, N, K, bits, group_size, dtype, 1,
                 1, stream);
        if (st != QMV_OK) return st;
    }
    return QMV_OK;
}

int qmv_affine_swiglu(const void* x, const void* w_gate, const void* s_gate, const void* b_gate, const void* w_up,
                      const void* s_up, const void* b_up, const float* route_weight, void* mid, int M, int N, int K,
                      int bits, int group_size, int dtype, float clamp, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (K % group_size != 0) return QMV_EINVAL;
    if (!(clamp >= 0.0f)) return QMV_EINVAL;                     // negative or NaN clamp
    st = check_common(x, w_gate, s_gate, mid, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    if (K > 0 && (!b_gate || !w_up || !s_up || !b_up)) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (K > 0 && (!aligned(w_up, 4) || !aligned(s_gate, eb) || !aligned(b_gate, eb) || !aligned(s_up, eb) ||
                  !aligned(b_up, eb)))
        return QMV_EALIGN;
    if (route_weight && !aligned(route_weight, 4)) return QMV_EALIGN;
    if ((long long)N * 2 > 0x7FFFFFFFLL) return QMV_EINVAL;
    return run_pair(x, w_gate, s_gate, b_gate, w_up, s_up, b_up, route_weight, mid, M, N, K, bits, group_size,
                    dtype, clamp, stream);
}

int qmv_affine_qkv(const void* x, const void* w_q, const void* s_q, const void* b_q, const void* w_k,
                   const void* s_k, const void* b_k, const void* w_v, const void* s_v, const void* b_v, void* y,
                   int M, int Nq, int Nkv, int K, int bits, int group_size, int dtype, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (Nq < 0 || Nkv < 0 || K % group_size != 0) return QMV_EINVAL;
    if ((long long)Nq + 2LL * Nkv > 0x7FFFFFFFLL) return QMV_EINVAL;
    const int N = Nq + 2 * Nkv;
    st = check_common(x, w_q, s_q, y, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    const void* w[3] = {w_q, w_k, w_v};
    const void* s[3] = {s_q, s_k, s_v};
    const void* b[3] = {b_q, b_k, b_v};
    const size_t eb = elem_bytes(dtype);
    if (K > 0) {
        for (int i = 0; i < 3; ++i) {
            const int n = i == 0 ? Nq : Nkv;
            if (n == 0) continue;
            if (!w[i] || !s[i] || !b[i]) return QMV_EINVAL;
            if (!aligned(w[i], 4) || !aligned(s[i], eb) || !aligned(b[i], eb)) return QMV_EALIGN;
        }
    }
    return run_qkv(x, w, s, b, y, M, Nq, Nkv, K, bits, group_size, dtype, stream);
}

int qmv_affine_rms_norm(const void* x, const void* gamma, float eps, const void* w_packed, const void* scales,
                        const void* biases, void* y, int M, int N, int K, int bits, int group_size, int dtype,
                        void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (K % group_size != 0) return QMV_EINVAL;
    if (!(eps >= 0.0f) || !(eps < 3.0e38f)) return QMV_EINVAL;        // negative, NaN or infinite
    st = check_common(x, w_packed, scales, y, M, N, K, dtype);
    if (st != QMV_OK || M == 0 || N == 0) return st;
    if (K > 0 && (!biases || !gamma)) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (K > 0 && (!aligned(scales, eb) || !aligned(biases, eb) || !aligned(gamma, eb))) return QMV_EALIGN;
    return run_rms_norm(x, gamma, eps, w_packed, scales, biases, y, M, N, K, bits, group_size, dtype, stream);
}

int qmv_qvm_affine(const void* x, const void* w_packed, const void* scales, const void* biases, void* y,
                   int M, int N, int K, int bits, int group_size, int dtype, void* workspace, void* stream) {
    int st = check_affine(bits, group_size);
    if (st != QMV_OK) return st;
    if (dtype != QMV_F32 && dtype != QMV_F16 && dtype != QMV_BF16) return QMV_EUNSUPPORTED;
    if (M < 0 || M > QMV_MAX_M || N < 0 || K < 0 || N % group_size != 0) return QMV_EINVAL;
    if (M == 0 || N == 0) return QMV_OK;
    if (!y || (K > 0 && (!x || !w_packed || !scales || !biases))) return QMV_EINVAL;
    const size_t eb = elem_bytes(dtype);
    if (!aligned(y, eb) || (x && !aligned(x, eb)) || (scales && !aligned(scales, eb)) ||
        (biases && !aligned(biases, eb)) || (w_packed && !aligned(w_packed, 16)) ||
        (workspace && !aligned(workspace, 16)))
        return QMV_EALIGN;
    return finish(qmv::launch_qvm_affine(bits, dtype, x, w_packed, scales, biases, y, workspace, M, N, K,
                                         group_size, static_cast<cudaStream_t>(stream)));
}

size_t qmv_qvm_workspace_bytes(int M, int N) {
    if (M < 0 || N < 0) return 0;
    return qmv::qvm_workspace_bytes(M, N);
}

const char* qmv_status_string(int status) {
    switch (status) {
        case QMV_OK: return "ok";
        case QMV_EINVAL: return "invalid argument";
        case QMV_EUNSUPPORTED: return "unsupported bits, group size, mode, dtype or size";
        case QMV_EALIGN: return "misaligned pointer";
        case QMV_ECUDA: return "CUDA launch error";
        default: return "unknown status";
    }
}

int qmv_last_cuda_error(void) { return g_last_cuda; }

int qmv_describe_plan(int family, int M, int N, int K, int bits, int group_size, int dtype, int w_align16,
                      char* buf, int buflen) {
    if (!buf || buflen <= 0) return QMV_EINVAL;
    if (M < 1 || M > QMV_QMM_MAX_M || N < 1 || K < 0) return QMV_EINVAL;
    int fam, G, fes = 1;
    if (family == 0) {
        if (check_affine(bits, group_size) != QMV_OK) return QMV_EUNSUPPORTED;
        fam = qmv::FAM_AFFINE;
        G = group_size;
    } else if (family >= 100) {
        if (family - 100 >= QMV_FMT_COUNT) return QMV_EUNSUPPORTED;
        const BsFmt& f = kBsFmt[family - 100];
        fam = f.fam; bits = f.bits; G = f.block;
        fes = scale_bytes_of(f.skind);
    } else {
        fam = fp_family(family - 1);
        if (fam < 0) return QMV_EUNSUPPORTED;
        bits = 0;
        G = family == 2 ? 16 : 32;
    }
    Plan pl;
    const bool qmm = M > QMV_MAX_M;
    if (qmm && fam != qmv::FAM_AFFINE) return QMV_EINVAL;
    int st = make_plan(fam, M, N, K, bits, G, dtype, w_align16 != 0, 1, &pl, true, false, false, true,
                       qmm && qmm_prefers_umma(M, N, K, bits, G, dtype, w_align16 != 0, true), false, false, fes);
    if (st != QMV_OK) return st;
    if (qmm && pl.tc != 5) {
        // qmm: chunks of x rows, each through the qmv plan of its size
        const int c = qmm_chunk(M, N, K, bits, group_size, dtype, w_align16 != 0, true);
        st = make_plan(fam, c, N, K, bits, group_size, dtype, w_align16 != 0, 1, &pl);
        if (st != QMV_OK) return st;
        snprintf(buf, (size_t)buflen, "path=chunked%d chunks=%d ", c, (M + c - 1) / c);
        const size_t n0 = strlen(buf);
        if ((int)n0 >= buflen) return QMV_OK;
        buf += n0;
        buflen -= (int)n0;
    }
    snprintf(buf, (size_t)buflen,
             "path=%s chunk=%d maxm=%d rows_per_warp=%d warps_k=%d warps_rows=%d tile_iters=%d "
             "grid=%u block=%u smem=%zu stage_sb=%d batch_sb=%d scale_ring=%d",
             pl.tc == 6 ? "tcg" : pl.tc == 5 ? "umma" : pl.tc == 4 ? "tcf" : pl.tc == 3 ? "direct" : pl.tc == 2 ? "tcb" : pl.tc ? "tc" : pl.wide ? "wide" : "narrow", pl.C, pl.maxm, pl.R, pl.wk, pl.wr,
             pl.tile_iters, pl.grid.x, pl.block.x, pl.smem, pl.sps, pl.spb, pl.sring);
    return QMV_OK;
}

int qmv_device_fault(unsigned int* code, int clear) {
    if (!code) return QMV_EINVAL;
    *code = 0;
    if (!fault_word()) return QMV_ECUDA;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_qmv_fault, sizeof(unsigned));
    if (e == cudaSuccess && clear) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_qmv_fault, &zero, sizeof(unsigned));
    }
    return finish(e);
}

void qmv_test_skip_last_copy(int enable) { g_test_skip.store(enable ? 1 : 0, std::memory_order_relaxed); }

void qmv_force_config(int path, int rows_per_warp, int warps_k, int warps_rows) {
    g_forced.path = path;
    g_forced.R = rows_per_warp;
    g_forced.wk = warps_k;
    g_forced.wr = warps_rows;
}

}  // extern "C"
