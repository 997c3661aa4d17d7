// qmv_umma.cuh -- affine qmv / small-M qmm on the 5th-generation tensor cores
// (tcgen05.mma, A from tensor memory, B from shared memory, fp32 accumulators
// in tensor memory), one bf16 x row up to 64.
//
// Why this shape.  The CUDA-core kernels spend about three instructions per
// code (decode, FMA, addressing); the mma.sync kernels issue their warp-level
// MMAs in order between the decode instructions.  Here a code costs one
// masked OR per PAIR plus one packed bf16 subtraction (qmv_tc_plan.cuh: the
// pair becomes {c_lo 2^s_lo, c_hi 2^s_hi} exactly), and the decoded pairs go
// straight from registers into TENSOR MEMORY with tcgen05.st, where the MMA
// reads them as its A operand: no shared-memory round trip for the decoded
// weights, and the MMAs are issued asynchronously by one thread.
//
// Tile: 128 weight rows x the CTA's K range; MMA M = 128 (lane = weight row),
// N = NCOL (16..64) x rows (x row m = MMA column m; columns past M are never
// read), K = 16 per instruction.
//
// Roles (one CTA per SM, persistent over row tiles):
//   warp 0     producer: the weight ring (one 3-D tensor copy per 128-byte
//              column box, 128-byte swizzle, rows past N zero-filled) and the
//              scale / bias ring (boxes of 8 groups x 128 rows); no multicast.
//   warp 1     allocates tensor memory; lane 0 issues the MMAs of each block
//              of codes once its A is written, and commits their completion.
//   warps 2-9  decoders: thread = weight row 32 (warp % 4) + lane (the tensor
//              memory lanes a warp may touch); half h = (warp - 2) / 4 takes the
//              blocks b = h, h + 2, ... of the K range.  A block is
//              max(group, 64) codes: its A slots (64 codes each) are decoded
//              into tensor memory, and DB blocks are in flight.  After the MMA
//              of a block completes, the same half reads its accumulator(s)
//              back (tcgen05.ld) and applies the group's scale and bias in fp32:
//                  y[m] += scale * D[m] + bias * sum(x[m] over the group),
//              sum(x) formed from values widened to fp32 one by one.
// B (x): the CTA's K range of x, staged once per CTA in the k-slot order of
// the decode plan (x~ = x * 2^(w - s), exact for bf16) in the canonical
// K-major no-swizzle layout, core matrix rows = x rows: element (m, slot t) at
// ((t / 8) * M + m) * 16 + (t % 8) * 2 bytes, so the descriptor's stride
// between 8-row groups is 128 bytes and between K halves 16 * M bytes.  Rows
// m >= M of the MMA read the next rows of that buffer (never-read columns).
// K split: the CTAs of a thread-block cluster (S <= 16) take contiguous K
// ranges of the same row tiles; their fp32 partials meet through distributed
// shared memory (each CTA sums a slice of the rows in rank order), so nothing
// outside the caller's buffers is written.
//
// Flow control: full / empty barriers for both rings; afull[s] (4 decoder
// warps per block) and dfull[s] (one MMA commit per block) for the block
// slots.  Every wait is bounded (about one second of %globaltimer); on expiry
// the kernel ORs a code into p.fault (1: a decoder gave up on a ring slot,
// 2: the producer on an empty slot, 4: the producer on its own copies, 8: the
// MMA thread on a block's A, 16: a decoder on a block's accumulator), stops
// its work and keeps every barrier schedule, so every thread ends.
#pragma once

#include <cuda_bf16.h>

#include "qmv_tcb.cuh"

namespace qmv {

// ---------------------------------------------------------- tcgen05 / TMEM --
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 8 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// N (1, 2, 4, 8, 16) consecutive fp32 columns of this thread's lane.
template <int N> __device__ __forceinline__ void tmem_ld(uint32_t taddr, float* v);
template <> __device__ __forceinline__ void tmem_ld<1>(uint32_t taddr, float* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=f"(v[0]) : "r"(taddr) : "memory");
}
template <> __device__ __forceinline__ void tmem_ld<2>(uint32_t taddr, float* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=f"(v[0]), "=f"(v[1]) : "r"(taddr)
                 : "memory");
}
template <> __device__ __forceinline__ void tmem_ld<4>(uint32_t taddr, float* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                 : "r"(taddr)
                 : "memory");
}
template <> __device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, float* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "r"(taddr)
                 : "memory");
}
template <> __device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, float* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
          "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr)
        : "memory");
}
template <int N> __device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float* v) {
    if constexpr (N <= 16) {
        tmem_ld<N>(taddr, v);
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 16) tmem_ld<16>(taddr + (uint32_t)i, v + i);
    }
}

// D[tmem] (+)= A[tmem] * B[smem desc]: kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// Shared-memory matrix descriptor, K-major, no swizzle: start address, the
// byte distance between the two 8-element K halves of a core matrix row set
// (lbo) and between 8-row groups (sbo); descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Generic-proxy shared-memory writes -> visible to the tensor cores' reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
// Waits that suspend: try_wait with a suspend-time hint parks the thread in
// hardware until the phase completes (or the hint runs out), so waiting warps
// take no issue slots from the decoders and the MMA thread.  (A plain
// try_wait loop returned at once and spun: measured on B200 it starved the
// SM's other warps, about 0.9 us per block of codes.)  Bounded by about one
// second, as every wait here.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool um_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// Arrive (release at cluster scope) on the mbarrier at the same shared
// address in the CTA of the given cluster rank.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t local_bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_bar), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
// Bounded wait (about one second) with cluster-scope acquire.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// ------------------------------------------------------------- geometry ----
// Per code width: unit = what one thread decodes at once (TcGeom), pairs per
// unit rounded up to 8 (one MMA K step is 8 pair columns), A slot = 64 codes.
template <int B> struct UmGeom {
    using Gm = TcGeom<B>;
    static constexpr int UC = Gm::UNIT_CODES, UB = Gm::UNIT_BYTES, NW = Gm::NW;
    static constexpr int NP = tc_make_plan<B, false>().np;
    static constexpr int NPU = (NP + 7) / 8 * 8;           // columns per unit
    static constexpr int SU = 64 / UC;                      // units per A slot
    static constexpr int SLOT_COLS = SU * NPU;              // columns per A slot
    static constexpr int KS64 = 2 * SLOT_COLS;              // k-slots per 64 codes
    // weight ring: stage = NBOX boxes of 128 bytes per row (a whole number of
    // units; 5-bit units are 20 bytes)
    static constexpr int NBOX = (B == 3 || B == 6) ? 3 : (B == 5) ? 5 : 2;
    static constexpr int SEGB = 128 * NBOX;                 // stage bytes per row
    static constexpr int STAGE_CODES = SEGB * 8 / B;
    static constexpr int STAGE_BYTES = 128 * SEGB;
    static_assert(SEGB % UB == 0 && STAGE_CODES % 64 == 0, "stage holds whole units and 64-code slots");
};

// The k-slot table of one unit: x code offset (-1: empty) and the exponent
// w - s that x is scaled by in that slot (slot 2p: low half of pair p, 2p + 1:
// its high half).
template <int B> struct UmXTab {
    int code[64];
    int ex[64];
};
template <int B> __host__ __device__ constexpr UmXTab<B> um_make_xtab() {
    constexpr TcPlanData P = tc_make_plan<B, false>();
    UmXTab<B> t{};
    for (int p = 0; p < UmGeom<B>::NPU; ++p) {
        for (int h = 0; h < 2; ++h) {
            const int f = p < P.np ? (h ? P.hi[p] : P.lo[p]) : -1;
            t.code[2 * p + h] = f < 0 ? -1 : tc_field_code<B>(f);
            t.ex[2 * p + h] = f < 0 ? 0 : tc_field_wexp<B>(f) - (h ? P.shi[p] : P.slo[p]);
        }
    }
    return t;
}

// Launch parameters of the tensor-memory kernel beyond Params.
struct UmmaParams {
    int S;            // K split = cluster size (1..16; beyond 8 non-portable)
    int DB;           // blocks in flight (even)
    int WST, SSL;     // weight stages, scale slots (<= 8 each)
    int nq, QC;       // K in quanta of QC codes (a range boundary)
    int ncols;        // tensor memory columns allocated (power of two)
    int ncol_mma;     // MMA N (16..64)
    int tiles;        // 128-row tiles
    unsigned smem_b;  // bytes reserved for B (x~) of one K range, tail included
    int ngr_max;      // groups of the longest K range: every CTA of a cluster
                      // lays out shared memory alike (peers read `red` at the
                      // same offset)
};

// The NPU pair registers of one unit (empty pairs and padding are 0).
template <int B, int NPU, int... Q>
__device__ __forceinline__ void um_pairs(std::integer_sequence<int, Q...>, const uint32_t (&w)[TcGeom<B>::NW],
                                         uint32_t kbf16, uint32_t (&a)[NPU]) {
    constexpr int NP = tc_make_plan<B, false>().np;
    ((a[Q] = (Q < NP) ? tc_pair<B, (Q < NP ? Q : 0)>(w, kbf16) : 0u), ...);
}

// y[m] += scale * D[m] + bias * sum(x[m]) for the NBG groups of one block.
template <int MLD>
__device__ __forceinline__ void um_epilogue(float (&y)[MLD], uint32_t dtaddr, int ncol_mma, int NBG,
                                            const float2* sb, const float* sxg, int ngr, int M) {
    for (int q = 0; q < NBG; ++q) {
        float d[MLD];
        tmem_ld_n<MLD>(dtaddr + (uint32_t)(q * ncol_mma), d);
        tmem_wait_ld();
        const float2 c = sb[q * 128];
#pragma unroll
        for (int m = 0; m < MLD; ++m)
            if (m < M) y[m] = fmaf(c.x, d[m], fmaf(c.y, sxg[q + (size_t)m * ngr], y[m]));
    }
}

// Shared memory (bytes; base rounded up to 1024, the host adds the slack):
//   0      barriers: wfull[8] wempty[8] sfull[8] sempty[8] afull[16] dfull[16]
//          cready cdone, and the tensor memory address at byte 1016
//   1024   weight ring: WST stages of STAGE_BYTES (NBOX swizzled boxes of
//          128 rows x 128 bytes)
//          scale ring: SSL slots of 4096 (scales then biases, 128 x 8 bf16)
//          B: x~ of the K range, smem_b bytes
//          sx: M x ngr_max floats (sum(x) per group), rounded up to 16 bytes
//          sbuf: DB x NBG x 128 float2 (scale, bias of blocks in flight)
//          red: 128 x MLD floats
template <int B, int MLD>
__global__ void __launch_bounds__(320, 1) qmv_umma_kernel(const __grid_constant__ Params p,
                                                           const __grid_constant__ UmmaParams u) {
    using Gm = UmGeom<B>;
    constexpr UmXTab<B> XT = um_make_xtab<B>();
    constexpr int UC = Gm::UC, UB = Gm::UB, NW = Gm::NW, NPU = Gm::NPU, SU = Gm::SU;
    constexpr int SLOT_COLS = Gm::SLOT_COLS, KS64 = Gm::KS64;
    constexpr int STAGE_CODES = Gm::STAGE_CODES, STAGE_BYTES = Gm::STAGE_BYTES, NBOX = Gm::NBOX;
    using T = __nv_bfloat16;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = p.M, N = p.N, K = p.K, G = p.G;
    const int S = u.S, DB = u.DB, WST = u.WST, SSL = u.SSL;
    const int rank = S > 1 ? (int)cluster_rank() : 0;
    const int q0 = (int)((long long)rank * u.nq / S), q1 = (int)((long long)(rank + 1) * u.nq / S);
    const int k0 = q0 * u.QC, k1 = min(K, q1 * u.QC);
    const int BLK = G > 64 ? G : 64;                  // codes per block
    const int NBG = BLK / G;                           // groups per block
    const int NBS = BLK / 64;                          // A slots per block
    const int nblk = (k1 - k0) / BLK;
    const int ngr = (k1 - k0) / G;
    const int nstage = (k1 - k0 + STAGE_CODES - 1) / STAGE_CODES;
    const int nsslot = (ngr + 7) / 8;
    const int UPG = G / UC;                            // units per group
    const int KSG = 2 * NPU * UPG;                     // k-slots per group
    const int ncl = gridDim.y;
    const int ntile_mine = u.tiles > (int)blockIdx.y ? (u.tiles - (int)blockIdx.y + ncl - 1) / ncl : 0;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 1016);
    unsigned char* wring = smem + 1024;
    unsigned char* sring = wring + (size_t)WST * STAGE_BYTES;
    unsigned char* xb = sring + (size_t)SSL * 4096;
    float* sx = reinterpret_cast<float*>(xb + u.smem_b);
    float2* sbuf = reinterpret_cast<float2*>(sx + (size_t)(M * u.ngr_max + 3) / 4 * 4);
    float* red = reinterpret_cast<float*>(sbuf + (size_t)DB * NBG * 128);
    const uint32_t bar0 = smem_addr(bars);
    auto wfull = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto wempty = [&](int s) { return bar0 + 8u * (uint32_t)(8 + s); };
    auto sfull = [&](int s) { return bar0 + 8u * (uint32_t)(16 + s); };
    auto sempty = [&](int s) { return bar0 + 8u * (uint32_t)(24 + s); };
    auto afull = [&](int s) { return bar0 + 8u * (uint32_t)(32 + s); };
    auto dfull = [&](int s) { return bar0 + 8u * (uint32_t)(48 + s); };
    const uint32_t cready = bar0 + 8u * 64u, cdone = bar0 + 8u * 65u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < WST; ++s) { mbar_init(wfull(s), 1); mbar_init(wempty(s), 8); }
        for (int s = 0; s < SSL; ++s) { mbar_init(sfull(s), 1); mbar_init(sempty(s), 8); }
        for (int s = 0; s < DB; ++s) { mbar_init(afull(s), 4); mbar_init(dfull(s), 1); }
        mbar_init(cready, (uint32_t)(256 * S));
        mbar_init(cdone, (uint32_t)(256 * S));
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), (uint32_t)u.ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (S > 1) cluster_sync_all();          // every CTA's barriers exist before any remote arrival
    const uint32_t tbase = *tmem_slot;
    const uint32_t dcol0 = (uint32_t)(DB * NBS * SLOT_COLS);
    bool ok = true;

    if (warp == 0) {
        // ===================== producer =====================================
        grid_launch_dependents();
        const uint32_t w0 = smem_addr(wring), s0 = smem_addr(sring);
        int ws = 0, ss = 0;
        for (int i = 0; i < ntile_mine; ++i) {
            const int row0 = ((int)blockIdx.y + i * ncl) * 128;
            int snext = 0;
            for (int st = 0; st < nstage; ++st) {
                const int glast = min(ngr, (st + 1) * STAGE_CODES / G) - 1;
                for (; snext <= glast / 8 && snext < nsslot; ++snext, ++ss) {
                    const int slot = ss % SSL, f = ss / SSL;
                    if (ok && f > 0 && !um_wait(sempty(slot), (uint32_t)((f - 1) & 1))) ok = false;
                    if (ok && lane == 0) {
                        mbar_arrive_expect_tx(sfull(slot), 4096u);
                        const int gx = k0 / G + 8 * snext;
                        tensor_copy_3d(s0 + (uint32_t)slot * 4096u, &p.smap, gx, row0, 0, sfull(slot));
                        tensor_copy_3d(s0 + (uint32_t)slot * 4096u + 2048u, &p.bmap, gx, row0, 0, sfull(slot));
                    }
                    __syncwarp();
                }
                const int slot = ws % WST, f = ws / WST;
                if (ok && f > 0 && !um_wait(wempty(slot), (uint32_t)((f - 1) & 1))) ok = false;
                if (ok && lane == 0) {
                    mbar_arrive_expect_tx(wfull(slot), (uint32_t)STAGE_BYTES);
                    const int xe = (int)((long long)(k0 + st * STAGE_CODES) * B / 64);     // u64 elements
#pragma unroll
                    for (int j = 0; j < NBOX; ++j)
                        tensor_copy_3d(w0 + (uint32_t)(slot * STAGE_BYTES + j * 16384), &p.wmap, xe + 16 * j, row0, 0,
                                       wfull(slot));
                }
                __syncwarp();
                ++ws;
            }
        }
        unsigned code = ok ? 0u : 2u;
        for (int s = 0; s < WST && s < ws; ++s) {
            const int g_ = ws - 1 - s;
            if (!um_wait(wfull(g_ % WST), (uint32_t)((g_ / WST) & 1))) code |= 4u;
        }
        for (int s = 0; s < SSL && s < ss; ++s) {
            const int g_ = ss - 1 - s;
            if (!um_wait(sfull(g_ % SSL), (uint32_t)((g_ / SSL) & 1))) code |= 4u;
        }
        if (code && lane == 0) atomicOr(p.fault, code);
    } else {
        // x and y may belong to the previous kernel in the stream
        grid_wait();
        // ===================== x staging (warps 1..9) =======================
        // B: x~ of the K range in k-slot order (16-byte core-matrix rows); sx:
        // sum(x) per (x row, group), widened per element.
        {
            const int nthr = 288, tid = threadIdx.x - 32;
            const T* X = reinterpret_cast<const T*>(p.x);
            for (int it = tid; it < M * ngr; it += nthr) {
                const int m = it / ngr, gi = it % ngr;
                float s = 0.f;
                for (int uu = 0; uu < UPG; ++uu) {
                    const T* xr = X + (long long)m * K + k0 + (long long)gi * G + uu * UC;
                    float v[UC];
#pragma unroll
                    for (int q = 0; q < UC / 8; ++q) {
                        const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(xr) + q);
                        widen8<T>(w4, v + 8 * q);
                    }
#pragma unroll
                    for (int j = 0; j < UC; ++j) s += v[j];
                    const int t8 = (gi * KSG + uu * 2 * NPU) >> 3;
#pragma unroll
                    for (int c8 = 0; c8 < 2 * NPU / 8; ++c8) {
                        uint32_t h[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int sl0 = 8 * c8 + 2 * e, sl1 = sl0 + 1;
                            const float lo = XT.code[sl0] >= 0
                                                 ? __fmul_rn(v[XT.code[sl0] < 0 ? 0 : XT.code[sl0]],
                                                             __uint_as_float((uint32_t)(127 + XT.ex[sl0]) << 23))
                                                 : 0.f;
                            const float hi = XT.code[sl1] >= 0
                                                 ? __fmul_rn(v[XT.code[sl1] < 0 ? 0 : XT.code[sl1]],
                                                             __uint_as_float((uint32_t)(127 + XT.ex[sl1]) << 23))
                                                 : 0.f;
                            h[e] = bf16_bits(lo) | (bf16_bits(hi) << 16);
                        }
                        *reinterpret_cast<uint4*>(xb + ((size_t)(t8 + c8) * M + m) * 16) =
                            make_uint4(h[0], h[1], h[2], h[3]);
                    }
                }
                sx[it] = s;
            }
            // the bytes past the last core matrix that MMA rows >= M read (never-read
            // columns, kept finite)
            uint32_t* tail = reinterpret_cast<uint32_t*>(xb + (size_t)(ngr * KSG / 8) * M * 16);
            for (int i = tid; i < 64 * 16 / 4; i += nthr) tail[i] = 0u;
            fence_proxy_async_smem();
            asm volatile("bar.sync 2, 288;" ::: "memory");
        }

        if (warp == 1) {
            // ===================== MMA issuer ===============================
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(u.ncol_mma >> 3) << 17) |
                                   ((uint32_t)(128 >> 4) << 24);
            const uint32_t xb_addr = smem_addr(xb);
            const uint32_t lbo = 16u * (uint32_t)M, sbo = 128u;
            constexpr int STEPS = SLOT_COLS / 8;                 // MMA K steps per A slot
            const int spg = (NBS * STEPS) / NBG;                 // K steps per group
            int gb = 0;
            for (int i = 0; i < ntile_mine; ++i) {
                for (int b = 0; b < nblk; ++b, ++gb) {
                    const int bs = gb % DB;
                    if (ok && !um_wait(afull(bs), (uint32_t)((gb / DB) & 1))) {
                        ok = false;
                        if (lane == 0) atomicOr(p.fault, 8u);
                    }
                    __syncwarp();
                    if (ok) {
                        tc_fence_after();
                        if (lane == 0) {
                            const uint32_t abase = tbase + (uint32_t)(bs * NBS * SLOT_COLS);
                            const uint32_t dbase = tbase + dcol0 + (uint32_t)(bs * NBG * u.ncol_mma);
                            const int kslot0 = b * NBG * KSG;
                            for (int step = 0; step < NBS * STEPS; ++step) {
                                const int q = step / spg;
                                const uint32_t kc = (uint32_t)((kslot0 + 16 * step) >> 3);   // 8-slot column
                                const uint64_t bd = smem_desc(xb_addr + kc * 16u * (uint32_t)M, lbo, sbo);
                                umma_bf16_ts(dbase + (uint32_t)(q * u.ncol_mma), abase + (uint32_t)(8 * step), bd,
                                             idesc, (step % spg) ? 1u : 0u);
                            }
                            umma_commit(dfull(bs));
                        }
                        __syncwarp();
                    }
                }
            }
            // the last commits complete before tensor memory is released
            for (int s = 0; s < DB && s < gb; ++s) {
                const int g_ = gb - 1 - s;
                if (!um_wait(dfull(g_ % DB), (uint32_t)((g_ / DB) & 1))) break;
            }
        } else {
            // ===================== decoders (warps 2..9) ===================
            const int q4 = warp & 3;
            const int half = (warp - 2) >> 2;
            const int r = q4 * 32 + lane;
            const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
            const uint32_t kbf16 = p.kbf16;
            const uint32_t w0 = smem_addr(wring);
            const uint32_t sw = (uint32_t)(r & 7) << 4;
            T* Y = reinterpret_cast<T*>(p.y);
            float y[MLD];
            int gb = 0, ws_cur = 0, ss_cur = 0, ws_base = 0, ss_base = 0;
            for (int i = 0; i < ntile_mine; ++i) {
                const int row0 = ((int)blockIdx.y + i * ncl) * 128;
#pragma unroll
                for (int m = 0; m < MLD; ++m) y[m] = 0.f;
                const int gbt = gb;
                auto epi = [&](int b) {
                    const int g = gbt + b, bs = g % DB;
                    if (ok && !um_wait(dfull(bs), (uint32_t)((g / DB) & 1))) {
                        ok = false;
                        if (lane == 0) atomicOr(p.fault, 16u);
                    }
                    __syncwarp();
                    if (!ok) return;
                    tc_fence_after();
                    um_epilogue<MLD>(y, tbase + lane_off + dcol0 + (uint32_t)(bs * NBG * u.ncol_mma), u.ncol_mma,
                                     NBG, sbuf + (size_t)bs * NBG * 128 + r, sx + b * NBG, ngr, M);
                };
                for (int b = half; b < nblk; b += 2) {
                    const int g = gbt + b, bs = g % DB;
                    if (b >= DB) epi(b - DB);
                    const int st = (b * BLK) / STAGE_CODES;
                    while (ws_cur < ws_base + st) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(wempty(ws_cur % WST));
                        ++ws_cur;
                    }
                    const int sl = (b * NBG) / 8;
                    while (ss_cur < ss_base + sl) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(sempty(ss_cur % SSL));
                        ++ss_cur;
                    }
                    if (ok && !um_wait(wfull(ws_cur % WST), (uint32_t)((ws_cur / WST) & 1))) {
                        ok = false;
                        if (lane == 0) atomicOr(p.fault, 1u);
                    }
                    if (ok && !um_wait(sfull(ss_cur % SSL), (uint32_t)((ss_cur / SSL) & 1))) {
                        ok = false;
                        if (lane == 0) atomicOr(p.fault, 1u);
                    }
                    __syncwarp();
                    if (ok) {
                        const unsigned short* sp =
                            reinterpret_cast<const unsigned short*>(sring + (size_t)(ss_cur % SSL) * 4096);
                        for (int q = 0; q < NBG; ++q) {
                            const int j = (b * NBG + q) & 7;
                            const float sc = __uint_as_float((uint32_t)sp[r * 8 + j] << 16);
                            const float bi = __uint_as_float((uint32_t)sp[1024 + r * 8 + j] << 16);
                            sbuf[((size_t)bs * NBG + q) * 128 + r] = make_float2(sc, bi);
                        }
                        const uint32_t rowb = w0 + (uint32_t)((ws_cur % WST) * STAGE_BYTES) + (uint32_t)(r * 128);
                        const int off0 = (int)(((long long)(b * BLK) % STAGE_CODES) * B / 8);
                        const uint32_t acol = tbase + lane_off + (uint32_t)(bs * NBS * SLOT_COLS);
#pragma unroll 1
                        for (int un = 0; un < NBS * SU; ++un) {
                            const int o = off0 + un * UB;
                            uint32_t wv[NW];
                            if constexpr (UB == 16) {
                                const uint32_t addr =
                                    rowb + (uint32_t)((o >> 7) * 16384) + ((((uint32_t)(o >> 4) & 7u) << 4) ^ sw);
                                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                             : "=r"(wv[0]), "=r"(wv[1]), "=r"(wv[2]), "=r"(wv[3])
                                             : "r"(addr));
                            } else {
#pragma unroll
                                for (int q = 0; q < NW; ++q) {
                                    const int ob = o + 4 * q;
                                    const uint32_t addr = rowb + (uint32_t)((ob >> 7) * 16384) +
                                                          (((((uint32_t)(ob >> 4) & 7u) << 4) ^ sw) | (uint32_t)(ob & 15));
                                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wv[q]) : "r"(addr));
                                }
                            }
                            uint32_t a[NPU];
                            um_pairs<B, NPU>(std::make_integer_sequence<int, NPU>{}, wv, kbf16, a);
#pragma unroll
                            for (int c = 0; c < NPU; c += 8) tmem_st8(acol + (uint32_t)(un * NPU + c), a + c);
                        }
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(afull(bs));
                }
                // drain: this half's blocks whose accumulators are still unread
                for (int b = half; b < nblk; b += 2)
                    if (b + DB >= nblk) epi(b);
                gb += nblk;
                while (ws_cur < ws_base + nstage) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(wempty(ws_cur % WST));
                    ++ws_cur;
                }
                while (ss_cur < ss_base + nsslot) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty(ss_cur % SSL));
                    ++ss_cur;
                }
                ws_base += nstage;
                ss_base += nsslot;

                // ---- the tile's outputs: halves, then the cluster's K ranges ----
                asm volatile("bar.sync 3, 256;" ::: "memory");
                if (half == 1) {
#pragma unroll
                    for (int m = 0; m < MLD; ++m) red[r * MLD + m] = y[m];
                }
                asm volatile("bar.sync 3, 256;" ::: "memory");
                if (half == 0) {
#pragma unroll
                    for (int m = 0; m < MLD; ++m) {
                        const float v = y[m] + red[r * MLD + m];
                        if (S > 1) red[r * MLD + m] = v;
                        else if (m < M && row0 + r < N) DT<T>::st(Y, (long long)m * N + row0 + r, v);
                    }
                }
                if (S > 1) {
                    // every rank's partial is in its `red`: signal all ranks, then
                    // each sums a slice of the rows over the ranks in order
                    for (int k = 0; k < S; ++k) mbar_arrive_remote(cready, (uint32_t)k);
                    if (ok && !mbar_wait_cluster(cready, (uint32_t)(i & 1))) {
                        ok = false;
                        if (lane == 0) atomicOr(p.fault, 32u);
                    }
                    if (ok) {
                        const int lo = rank * 128 / S, hi = (rank + 1) * 128 / S;
                        const uint32_t red_addr = smem_addr(red);
                        for (int e = threadIdx.x - 64; e < (hi - lo) * M; e += 256) {
                            const int rr = lo + e / M, m = e % M;
                            float v = 0.f;
                            for (int k = 0; k < S; ++k)
                                v += ld_dsmem_f32(red_addr + (uint32_t)(rr * MLD + m) * 4u, (uint32_t)k);
                            if (row0 + rr < N) DT<T>::st(Y, (long long)m * N + row0 + rr, v);
                        }
                    }
                    for (int k = 0; k < S; ++k) mbar_arrive_remote(cdone, (uint32_t)k);
                    if (ok && !mbar_wait_cluster(cdone, (uint32_t)(i & 1))) {
                        ok = false;
                        if (lane == 0) atomicOr(p.fault, 32u);
                    }
                } else {
                    asm volatile("bar.sync 3, 256;" ::: "memory");
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, (uint32_t)u.ncols);
}

}  // namespace qmv
