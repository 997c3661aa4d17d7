// qmv_tcb.cuh -- tensor-core affine qmv whose weights stream through a
// shared-memory ring filled by the tensor-copy engine (cp.async.bulk.tensor)
// under mbarrier flow control: one producer warp, wr x wk consumer warps.
//
// Why: the register-prefetch kernel (qmv_tc.cuh) keeps only a few KB per SM in
// flight, bounded by registers and occupancy, and stalls on load latency.  Here
// the bytes in flight are STAGES ring stages per SM (tens of KB), independent
// of the consumers' registers.
//
// Work: the grid is persistent over ROW BLOCKS of ROWS = 16*wr rows (block b
// takes row blocks b, b + gridDim.x, ...).  A row block's packed rows are cut
// along K into ring STAGES of S super-blocks; the producer copies stage after
// stage (the packed rows, and when their layout allows the stage's scales and
// biases: one 3-D tensor copy each) into the ring, across row-block
// boundaries, while consumers compute.  Consumer warp (wrid, wkid) owns row
// tile wrid (16 rows) and the super-blocks wkid, wkid + wk, ... of every
// stage, taken SPB at a time: one BATCH fills the 8*NPASS slot columns of the
// MMAs (decode and slot columns as in qmv_tc.cuh) and ends in one exact fp32
// epilogue.  Everything a lane needs to place its x fragments, scales and sums
// inside a batch is computed once per kernel, so a full batch runs without
// per-super-block index arithmetic or predicates; only the last, partial
// batch of a row takes the guarded path.
//
// Flow control: full[s] (one producer arrival + the copies' byte count) and
// empty[s] (one arrival per consumer warp).  Every wait is bounded (about one
// second of %globaltimer); on expiry the kernel ORs a code into the fault word
// p.fault (1: a consumer gave up on a full stage, 2: the producer gave up on an
// empty stage, 4: the producer gave up waiting for its own copies), stops
// computing, keeps its barrier schedule so no warp waits on another forever,
// and the producer waits (bounded) for every copy it issued before it exits.
//
// Ring rows are dense (pitch = the stage's S * 4 * UB bytes, as the tensor copy
// lays them out); the two rows one load instruction touches per 8 lanes then
// share banks, a 2-way conflict on the two unit loads per super-block.
#pragma once

#include <type_traits>

#include "qmv_tc.cuh"

namespace qmv {

// ----------------------------------------------------- mbarrier / bulk copy --
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s

// Wait for the phase of the given parity to complete; false after the limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}
// Tensor tile [box] of a 3-D tensor map -> this CTA's shared memory (128-byte
// aligned destination), completion counted on `bar` in bytes (the full box,
// out-of-range elements zero-filled).  No multicast.
__device__ __forceinline__ void tensor_copy_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                               uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}
// Barrier over the consumer warps only (named barrier 1).
__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}
// Adds one to a shared arrival counter, ordered after this thread's (and,
// through a preceding __syncwarp, its warp's) earlier shared-memory accesses
// and before its later ones; returns the previous count.
__device__ __forceinline__ unsigned arrive_count(unsigned* ctr) {
    unsigned old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(smem_addr(ctr)) : "memory");
    return old;
}

// Scale / bias element of a ring row (x dtype), widened to fp32.
template <class T> __device__ __forceinline__ float ring_scale(const unsigned char* row, int i);
template <> __device__ __forceinline__ float ring_scale<float>(const unsigned char* row, int i) {
    return reinterpret_cast<const float*>(row)[i];
}
template <> __device__ __forceinline__ float ring_scale<__half>(const unsigned char* row, int i) {
    return __half2float(reinterpret_cast<const __half*>(row)[i]);
}
template <> __device__ __forceinline__ float ring_scale<__nv_bfloat16>(const unsigned char* row, int i) {
    return __uint_as_float((uint32_t)reinterpret_cast<const unsigned short*>(row)[i] << 16);
}

// Shared memory (bytes, in order):
//   bars  128            full[STAGES], empty[STAGES] (8 bytes each)
//   ring  STAGES stages (128-byte aligned) of: ROWS packed rows (pitch bytes
//         each, dense), then (p.sring) the scale tile at p.soff and the bias
//         tile at p.boff, ROWS x p.sbw bytes each
//   xs    NSPLIT * plane * 4    plane = M*xrow + 4*NP + 4 u32: the x rows of
//                               the tile (bf16 pairs, fragment order), then one
//                               super-block of zeros read by inactive lanes
//   sxx   M * NSEG float2      {sum(x), sum(x~)} per segment of the tile
//   us    M * TU * 2 floats    per-unit sums
//   red   NCW * 16 * 8*NPASS floats
// MAXT: threads per block the kernel is compiled for, 32 * (wk * wr + 1) with
// wk * wr in {8, 12} consumer warps plus the producer warp (the register
// budget follows).
template <int B, class T, int NPASS, int SPB, int STAGES, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) qmv_tcb_kernel(const __grid_constant__ Params p) {
    using Gm = TcGeom<B>;
    constexpr TcPlanData P = tc_make_plan<B, false>();
    constexpr int NP = P.np, NSTEP = NP / 2;
    constexpr int NW = Gm::NW, UB = Gm::UNIT_BYTES, UC = Gm::UNIT_CODES, SB = Gm::SB;
    constexpr int NSPLIT = TcSplit<T>::n;
    constexpr int ES = (int)sizeof(T);
    static_assert(2 * STAGES * 8 <= 128, "barrier area");

    extern __shared__ float4 smem4[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(smem4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wk = p.wk, wr = p.wr, NCW = wk * wr;
    const int M = p.M;
    const int ROWS = 16 * wr;
    const int nrb = (p.N + ROWS - 1) / ROWS;
    const int NSBK = p.K / SB;
    const int S = p.sps;
    const int pitch = p.pitch;
    const int sbw = p.sbw;
    const bool sring = p.sring != 0;
    const int stage_bytes = ROWS * pitch + (sring ? 2 * ROWS * sbw : 0);
    const int TSB = p.tile_iters;
    const int TU = TSB * 4;
    const int G = p.G;
    const int segsz = min(G, SB);
    const int NGS = SB / segsz;
    const long long KG = p.K / G;
    const int xrow = TU * NP + 4;
    const int plane = M * xrow + 4 * NP + 4;
    const int NSEG = TSB * NGS;
    const int bz = blockIdx.z;
    // groups of a super-block: SB / G (G <= SB) or one per G / SB super-blocks
    const int gmul = G < SB ? __ffs(SB / G) - 1 : 0;
    const int gdiv = G > SB ? __ffs(G / SB) - 1 : 0;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    // ring on a 128-byte boundary (tensor-copy destinations); the host adds
    // 128 bytes of slack for this
    unsigned char* ring = smem + 128 + ((128u - (smem_addr(smem) & 127u)) & 127u);
    uint32_t* xs = reinterpret_cast<uint32_t*>(ring + (size_t)STAGES * stage_bytes);
    float2* sxx = reinterpret_cast<float2*>(xs + (size_t)NSPLIT * plane);
    float* us = reinterpret_cast<float*>(sxx + (size_t)M * NSEG);
    float* red = us + (size_t)M * TU * 2;
    const uint32_t bar0 = smem_addr(bars);
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(STAGES + s); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), (uint32_t)NCW);
        }
        mbar_init_fence();
    }
    __syncthreads();

    const long long sb0 = bz * p.s_bs;
    const int nks = (NSBK + S - 1) / S;
    // this block's stages: j = (i-th row block of the block) * nks + K stage
    // ---- producer warp: streams weights only, so it starts at once ---------
    // (written out here, not as a helper taking the tensor maps' addresses:
    // that form measured up to 25 % slower on B200 for the whole kernel)
    if (warp == NCW) {
        grid_launch_dependents();    // the next kernel may start fetching its weights
        const uint32_t ring0 = smem_addr(ring);
        const uint32_t stage_tx = (uint32_t)ROWS * ((uint32_t)pitch + (sring ? 2u * (uint32_t)sbw : 0u));
        int it = 0;
        bool ok = true;
        for (int rb = blockIdx.x; rb < nrb && ok; rb += gridDim.x) {
            for (int ks = 0; ks < nks; ++ks) {
                const int slot = it % STAGES, f = it / STAGES;
                if (f > 0 && !mbar_wait(empty(slot), (uint32_t)((f - 1) & 1))) { ok = false; break; }
                const uint32_t st0 = ring0 + (uint32_t)(slot * stage_bytes);
                // test hook (qmv_test_skip_last_copy): block (0, 0)'s final stage
                // gets neither its expected-bytes arrival nor its copies, so the
                // bounded waits on it run out (codes 1 and 4); no copy is left
                // in flight
                const bool skip = p.test_skip && blockIdx.x == 0 && blockIdx.z == 0 &&
                                  rb + (int)gridDim.x >= nrb && ks == nks - 1;
                if (lane == 0 && !skip) {
                    // one tensor copy each: the stage's packed rows (ROWS x pitch
                    // bytes), scale tile and bias tile (ROWS x sbw bytes); rows
                    // past N and columns past the row end are zero-filled and
                    // count in full
                    mbar_arrive_expect_tx(full(slot), stage_tx);
                    tensor_copy_3d(st0, &p.wmap, (ks * S * 4 * UB) / 8, rb * ROWS, bz, full(slot));
                    if (sring) {
                        const int g0 = ((ks * S) << gmul) >> gdiv;
                        tensor_copy_3d(st0 + (uint32_t)p.soff, &p.smap, g0, rb * ROWS, bz, full(slot));
                        tensor_copy_3d(st0 + (uint32_t)p.boff, &p.bmap, g0, rb * ROWS, bz, full(slot));
                    }
                }
                __syncwarp();
                ++it;
            }
        }
        unsigned code = ok ? 0u : 2u;
        // wait for the copies this warp issued: the last fill of each slot
        for (int s = 0; s < STAGES && s < it; ++s) {
            const int last = (it - 1 - s) / STAGES;
            if (!mbar_wait(full(s), (uint32_t)(last & 1))) code |= 4u;
        }
        if (code && lane == 0) atomicOr(p.fault, code);
        return;
    }

    // ---- consumer warps: x and y may belong to the previous kernel ---------
    grid_wait();
    const int nthr = NCW * 32;
    const int g = lane >> 2, t = lane & 3;
    const int wkid = warp % wk, wrid = warp / wk;
    const T* X = reinterpret_cast<const T*>(p.x) + bz * p.x_bs;

    // zero super-block of every plane (never overwritten by the x staging)
    for (int i = threadIdx.x; i < 4 * NP; i += nthr)
#pragma unroll
        for (int sp = 0; sp < NSPLIT; ++sp) xs[(size_t)sp * plane + (size_t)M * xrow + i] = 0u;

    // ---- per-lane slot geometry, fixed for the kernel ------------------------
    // Slot column j of pass pp (j = 8 pp + column) is (super-block sbi of the
    // batch, segment gs, x row m):  j = (sbi * NGS + gs) * M + m.
    const int per_sb = NGS * M;
    const int nslots = SPB * per_sb;
    const int useg = (t * UC) / segsz;            // segment of this lane's unit
    // B operand: the lane supplies x of slot column g; active in the batch's
    // super-block bi iff that slot belongs to (bi, useg).  Offsets are relative
    // to the batch's first super-block; xact multiplies the batch advance.
    int xo[NPASS][SPB], xact[NPASS][SPB];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp) {
        const int j = 8 * pp + g;
        const int m = j % M, q = j / M, gs = q % NGS, sbi = q / NGS;
#pragma unroll
        for (int bi = 0; bi < SPB; ++bi) {
            const bool a = j < nslots && gs == useg && sbi == bi;
            xact[pp][bi] = a ? 1 : 0;
            xo[pp][bi] = a ? m * xrow + (bi * wk * 4 + t) * NP : M * xrow + t * NP;
        }
    }
    // D / Y elements: column 8 pp + 2 t + c, rows g (e = c) and g + 8 (e = 2 + c)
    int dsb[NPASS][2];      // super-block of the slot within the batch (0 if unused)
    int dseg[NPASS][2];     // sxx offset: m * NSEG + sbi * wk * NGS + gs
    int dgrp[NPASS][2];     // super-block offset of the slot within the batch: sbi * wk
    int dgs[NPASS][2];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int j = 8 * pp + 2 * t + c;
            const int m = j % M, q = j / M;
            const int gs = q % NGS, sbi = j < nslots ? q / NGS : 0;
            dsb[pp][c] = j < nslots ? sbi : SPB;   // SPB: never present
            dseg[pp][c] = (j < nslots ? m : 0) * NSEG + sbi * wk * NGS + gs;
            dgrp[pp][c] = sbi * wk;
            dgs[pp][c] = gs;
        }

    const uint32_t kbf16 = p.kbf16;
    const bool pairc = (M & 1) == 0;   // even M: both columns of a lane in one slot group
    int it = 0;
    bool ok = true;
    bool x_whole = false;            // x of the whole K is staged (one tile)
    T* Yo = reinterpret_cast<T*>(p.y) + bz * p.y_bs;

    for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
        const int row0 = rb * ROWS + wrid * 16;
        const int rg = min(row0 + g, p.N - 1), rh = min(row0 + g + 8, p.N - 1);
        const T* scg = reinterpret_cast<const T*>(p.scales) + sb0 + (long long)rg * KG;
        const T* sch = reinterpret_cast<const T*>(p.scales) + sb0 + (long long)rh * KG;
        const T* big = reinterpret_cast<const T*>(p.biases) + sb0 + (long long)rg * KG;
        const T* bih = reinterpret_cast<const T*>(p.biases) + sb0 + (long long)rh * KG;

        float Y[NPASS][4];
#pragma unroll
        for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
            for (int e = 0; e < 4; ++e) Y[pp][e] = 0.f;

        for (int t0 = 0; t0 < NSBK; t0 += TSB) {
            const int tn = min(TSB, NSBK - t0);
            if (!x_whole) {
                // ---- stage x: fragment-ordered bf16 planes + per-unit sums ----
                consumer_sync(nthr);            // the previous tile is no longer read
                const int items = M * tn * 4;
                for (int it2 = threadIdx.x; it2 < items; it2 += nthr) {
                    const int m = it2 / (tn * 4), u = it2 - m * (tn * 4);
                    const long long k0 = (long long)t0 * SB + (long long)u * UC;
                    const T* xr = X + (long long)m * p.K + k0;
                    float xv[UC];
                    if constexpr (sizeof(T) == 2 && UC % 8 == 0) {
                        if (p.x_vec) {
#pragma unroll
                            for (int q = 0; q < UC / 8; ++q)
                                widen8<T>(__ldg(reinterpret_cast<const uint4*>(xr) + q), xv + 8 * q);
                        } else {
#pragma unroll
                            for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                        }
                    } else if constexpr (sizeof(T) == 4 && UC % 4 == 0) {
                        if (p.x_vec) {
#pragma unroll
                            for (int q = 0; q < UC / 4; ++q) {
                                const float4 f4 = __ldg(reinterpret_cast<const float4*>(xr) + q);
                                xv[4 * q] = f4.x; xv[4 * q + 1] = f4.y; xv[4 * q + 2] = f4.z; xv[4 * q + 3] = f4.w;
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                    }
                    float usum = 0.f;                  // sum(x), widened element by element
#pragma unroll
                    for (int c = 0; c < UC; ++c) usum += xv[c];
                    float tsum = 0.f;                  // sum of the fragment values x~
                    uint32_t* dst = xs + (size_t)m * xrow + (size_t)u * NP;
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        float lo = 0.f, hi = 0.f;
                        if (P.lo[q] >= 0)
                            lo = __fmul_rn(xv[tc_field_code<B>(P.lo[q])],
                                           __uint_as_float((uint32_t)(127 + tc_field_wexp<B>(P.lo[q]) - P.slo[q]) << 23));
                        if (P.hi[q] >= 0)
                            hi = __fmul_rn(xv[tc_field_code<B>(P.hi[q])],
                                           __uint_as_float((uint32_t)(127 + tc_field_wexp<B>(P.hi[q]) - P.shi[q]) << 23));
                        tsum += lo + hi;
#pragma unroll
                        for (int sp = 0; sp < NSPLIT; ++sp) {
                            const uint32_t bl = bf16_bits(lo), bh = bf16_bits(hi);
                            dst[(size_t)sp * plane + q] = bl | (bh << 16);
                            lo = lo - __uint_as_float(bl << 16);     // exact remainders
                            hi = hi - __uint_as_float(bh << 16);
                        }
                    }
                    us[((size_t)m * TU + u) * 2] = usum;
                    us[((size_t)m * TU + u) * 2 + 1] = tsum;
                }
                consumer_sync(nthr);
                const int upseg = segsz / UC;
                const int nseg = tn * NGS;
                for (int i = threadIdx.x; i < M * nseg; i += nthr) {
                    const int m = i / nseg, sg = i - m * nseg;
                    const float* ur = us + ((size_t)m * TU + (size_t)sg * upseg) * 2;
                    float a = 0.f, b = 0.f;
                    for (int q = 0; q < upseg; ++q) { a += ur[2 * q]; b += ur[2 * q + 1]; }
                    sxx[(size_t)m * NSEG + sg] = make_float2(a, b);
                }
                consumer_sync(nthr);
                x_whole = (TSB >= NSBK);
            }

            // ---- one batch: SPB super-blocks of this warp, then the epilogue ---
            // FULL: all SPB super-blocks exist (no guards); otherwise nex of them.
            // RING: scales and biases from the stage's tiles (sp: scale row g,
            // scale row g + 8, bias row g, bias row g + 8, each indexed by the
            // group within the stage), else from global memory (indexed by the
            // group within the row).  With an even M the two columns of a lane
            // share their slot's group: its scales are loaded once.
            auto run_batch = [&](auto full_c, auto ring_c, int sbf, int nex, int sbase, const unsigned char* rowg,
                                 const unsigned char* rowh, const unsigned char* const (&sp)[4]) {
                constexpr bool FULL = decltype(full_c)::value;
                constexpr bool RING = decltype(ring_c)::value;
                float sc[NPASS][4], bs[NPASS][4];
                const int a0 = RING ? sbf - sbase : sbf;
#pragma unroll
                for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        if (c == 1 && pairc) {
                            sc[pp][1] = sc[pp][0]; sc[pp][3] = sc[pp][2]; bs[pp][1] = bs[pp][0]; bs[pp][3] = bs[pp][2];
                            continue;
                        }
                        const bool pres = FULL || dsb[pp][c] < nex;
                        const int gi = (((a0 + dgrp[pp][c]) << gmul) >> gdiv) + dgs[pp][c];
                        float s0 = 0.f, s1 = 0.f, b0 = 0.f, b1 = 0.f;
                        if (pres) {
                            if constexpr (RING) {
                                s0 = ring_scale<T>(sp[0], gi); s1 = ring_scale<T>(sp[1], gi);
                                b0 = ring_scale<T>(sp[2], gi); b1 = ring_scale<T>(sp[3], gi);
                            } else {
                                s0 = DT<T>::ld(scg, gi); s1 = DT<T>::ld(sch, gi);
                                b0 = DT<T>::ld(big, gi); b1 = DT<T>::ld(bih, gi);
                            }
                        }
                        sc[pp][c] = s0; sc[pp][2 + c] = s1; bs[pp][c] = b0; bs[pp][2 + c] = b1;
                    }
                float D[NPASS][4], E[NPASS][4];     // two MMA chains (even / odd k-steps)
#pragma unroll
                for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                    for (int e = 0; e < 4; ++e) { D[pp][e] = 0.f; E[pp][e] = 0.f; }
                const int xadv = (sbf - t0) * 4 * NP;
#pragma unroll
                for (int bi = 0; bi < SPB; ++bi) {
                    if (FULL || bi < nex) {
                        const int uo = (sbf - sbase + bi * wk) * 4 * UB + t * UB;
                        uint32_t wg[NW], wh[NW];
                        if constexpr (UB == 16) {
                            const uint4 a = *reinterpret_cast<const uint4*>(rowg + uo);
                            const uint4 b = *reinterpret_cast<const uint4*>(rowh + uo);
                            wg[0] = a.x; wg[1] = a.y; wg[2] = a.z; wg[3] = a.w;
                            wh[0] = b.x; wh[1] = b.y; wh[2] = b.z; wh[3] = b.w;
                        } else {
#pragma unroll
                            for (int q = 0; q < NW; ++q) {
                                wg[q] = reinterpret_cast<const uint32_t*>(rowg + uo)[q];
                                wh[q] = reinterpret_cast<const uint32_t*>(rowh + uo)[q];
                            }
                        }
                        int xoff[NPASS];
#pragma unroll
                        for (int pp = 0; pp < NPASS; ++pp) xoff[pp] = xo[pp][bi] + xact[pp][bi] * xadv;
                        tc_steps2<B, NPASS, NSPLIT>(std::make_integer_sequence<int, NSTEP / 2>{}, wg, wh, D, E, xs,
                                                    xoff, plane, kbf16);
                    }
                }
                const int segadv = (sbf - t0) * NGS;
#pragma unroll
                for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float2 ab = make_float2(0.f, 0.f);
                        if (FULL || dsb[pp][c] < nex) ab = sxx[dseg[pp][c] + segadv];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int e = 2 * h + c;
                            Y[pp][e] = fmaf(sc[pp][e], D[pp][e] + E[pp][e], fmaf(bs[pp][e], ab.x, Y[pp][e]));
                        }
                    }
            };

            // ---- this warp's super-blocks of the tile, stage by stage -------
            const int end = t0 + tn;
            for (int ks = t0 / S; ks * S < end; ++ks) {
                const int slot = it % STAGES, f = it / STAGES;
                if (ok && !mbar_wait(full(slot), (uint32_t)(f & 1))) {
                    ok = false;
                    if (lane == 0) atomicOr(p.fault, 1u);
                }
                const int sbase = ks * S;
                const int send = min(end, sbase + S);
                if (ok) {
                    const unsigned char* rowg = ring + (size_t)slot * stage_bytes + (size_t)(wrid * 16 + g) * pitch;
                    const unsigned char* rowh = rowg + 8 * pitch;
                    // scale / bias tile rows of this lane: stage + offset + row * sbw
                    const unsigned char* tileg = ring + (size_t)slot * stage_bytes + (size_t)(wrid * 16 + g) * sbw;
                    const unsigned char* const sp[4] = {tileg + p.soff, tileg + p.soff + 8 * sbw, tileg + p.boff,
                                                        tileg + p.boff + 8 * sbw};
                    auto batches = [&](auto ring_c) {
                        for (int sbf = sbase + wkid; sbf < send; sbf += SPB * wk) {
                            if (sbf + (SPB - 1) * wk < send) {
                                run_batch(std::true_type{}, ring_c, sbf, SPB, sbase, rowg, rowh, sp);
                            } else {
                                const int nex = (send - sbf + wk - 1) / wk;
                                run_batch(std::false_type{}, ring_c, sbf, nex, sbase, rowg, rowh, sp);
                            }
                        }
                    };
                    if (sring) batches(std::true_type{});
                    else batches(std::false_type{});
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(slot));
                ++it;
            }
        }

        // ---- reduce over slots of the same x row and over k-warps, store -----
        // (every consumer takes a share: a reduction done by the last warp
        // alone measured up to 2x slower, it lands on the critical path)
        float* myred = red + (size_t)warp * 16 * 8 * NPASS;
#pragma unroll
        for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
            for (int e = 0; e < 4; ++e) myred[(g + 8 * (e >> 1)) * 8 * NPASS + 8 * pp + 2 * t + (e & 1)] = Y[pp][e];
        consumer_sync(nthr);
        const int tot = wr * 16 * M;
        for (int i = threadIdx.x; i < tot; i += nthr) {
            const int w_ = i / (16 * M), rm = i % (16 * M), r = rm / M, m = rm % M;
            const int row = rb * ROWS + w_ * 16 + r;
            float v = 0.f;
            for (int k = 0; k < wk; ++k) {
                const float* rr = red + (size_t)(w_ * wk + k) * 16 * 8 * NPASS + r * 8 * NPASS;
                for (int j = m; j < nslots; j += M) v += rr[j];
            }
            if (row < p.N) DT<T>::st(Yo, (long long)m * p.N + row, v);
        }
        consumer_sync(nthr);
    }

}

}  // namespace qmv
