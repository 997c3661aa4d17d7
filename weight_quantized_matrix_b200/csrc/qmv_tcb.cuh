// qmv_tcb.cuh -- tensor-core affine qmv whose weights stream through a
// shared-memory ring filled by the bulk-copy engine (cp.async.bulk) under
// mbarrier flow control: one producer warp, wr x wk consumer warps.
//
// Why: the register-prefetch kernel (qmv_tc.cuh) keeps only a few KB per SM in
// flight, bounded by registers and occupancy, and stalls on load latency.  Here
// the bytes in flight are STAGES ring stages per SM (tens of KB), independent
// of the consumers' registers.
//
// Work: the grid is persistent over ROW BLOCKS of ROWS = 16*wr rows (block b
// takes row blocks b, b + gridDim.x, ...).  A row block's packed rows are cut
// along K into STAGES of S super-blocks; the producer copies stage after stage
// (one bulk copy per row, issued by the producer's lanes) into the ring, across
// row-block boundaries, while consumers compute.  Consumer warp (wrid, wkid)
// owns row tile wrid (16 rows) and the super-blocks wkid, wkid + wk, ... of
// every stage; the decode, the slot-column MMAs and the exact per-group fp32
// epilogue are those of qmv_tc.cuh.
//
// Flow control: full[s] (one producer arrival + the copies' byte count) and
// empty[s] (one arrival per consumer warp).  Every wait is bounded (about one
// second of %globaltimer); on expiry the kernel ORs a code into the fault word
// p.fault (1: a consumer gave up on a full stage, 2: the producer gave up on an
// empty stage, 4: the producer gave up waiting for its own copies), stops
// computing, keeps its barrier schedule so no warp waits on another forever,
// and the producer waits (bounded) for every copy it issued before it exits.
//
// Ring rows are padded (pitch = 64 mod 128 bytes for 16-byte units, 16 mod
// 128 for 12/20-byte units) so the 8 rows read by one load instruction fall in
// distinct banks.
#pragma once

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
// Global -> this CTA's shared memory, completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// Barrier over the consumer warps only (named barrier 1).
__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Shared memory (bytes, in order):
//   bars  128            full[STAGES], empty[STAGES]
//   ring  STAGES * ROWS * pitch
//   xs    NSPLIT * plane * 4    plane = M*xrow + 4*NP + 4 u32: the x rows of
//                               the tile (bf16 pairs, fragment order), then one
//                               super-block of zeros read by inactive lanes
//   sx    M * NSEG floats        sum(x) per segment of the tile
//   sxt   M * NSEG floats        sum(x~) per segment
//   us    M * TU * 2 floats      per-unit sums
//   red   NCW * 16 * 8*NPASS floats
template <int B, class T, int NPASS, int STAGES>
__global__ void __launch_bounds__(288, 1) qmv_tcb_kernel(const Params p) {
    using Gm = TcGeom<B>;
    constexpr TcPlanData P = tc_make_plan<B, false>();
    constexpr int NP = P.np, NSTEP = NP / 2;
    constexpr int NW = Gm::NW, UB = Gm::UNIT_BYTES, UC = Gm::UNIT_CODES, SB = Gm::SB;
    constexpr int NSPLIT = TcSplit<T>::n;
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
    const int stage_bytes = ROWS * pitch;
    const int TSB = p.tile_iters;
    const int TU = TSB * 4;
    const int segsz = min(p.G, SB);
    const int NGS = SB / segsz;
    const int G = p.G;
    const long long KG = p.K / G;
    const int xrow = TU * NP + 4;
    const int plane = M * xrow + 4 * NP + 4;
    const int NSEG = TSB * NGS;
    const int bz = blockIdx.z;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    unsigned char* ring = smem + 128;
    uint32_t* xs = reinterpret_cast<uint32_t*>(ring + (size_t)STAGES * stage_bytes);
    float* sx = reinterpret_cast<float*>(xs + (size_t)NSPLIT * plane);
    float* sxt = sx + (size_t)M * NSEG;
    float* us = sxt + (size_t)M * NSEG;
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
    grid_wait();

    const uint8_t* W = p.w + bz * p.w_bs;
    const int nks = (NSBK + S - 1) / S;

    // ============================ producer warp ==============================
    if (warp == NCW) {
        const uint32_t ring0 = smem_addr(ring);
        int it = 0;
        bool ok = true;
        for (int rb = blockIdx.x; rb < nrb && ok; rb += gridDim.x) {
            for (int ks = 0; ks < nks; ++ks) {
                const int slot = it % STAGES, f = it / STAGES;
                if (f > 0 && !mbar_wait(empty(slot), (uint32_t)((f - 1) & 1))) { ok = false; break; }
                const int nsb = min(S, NSBK - ks * S);
                const uint32_t rowb = (uint32_t)(nsb * 4 * UB);
                if (lane == 0) mbar_arrive_expect_tx(full(slot), (uint32_t)ROWS * rowb);
                __syncwarp();
                for (int r = lane; r < ROWS; r += 32) {
                    const int row = min(rb * ROWS + r, p.N - 1);
                    bulk_copy_g2s(ring0 + (uint32_t)(slot * stage_bytes + r * pitch),
                                  W + (long long)row * p.w_row + (long long)ks * S * 4 * UB, rowb, full(slot));
                }
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
        grid_launch_dependents();
        return;
    }

    // ============================ consumer warps ============================
    const int nthr = NCW * 32;
    const int g = lane >> 2, t = lane & 3;
    const int wkid = warp % wk, wrid = warp / wk;
    const T* X = reinterpret_cast<const T*>(p.x) + bz * p.x_bs;
    const long long sb0 = bz * p.s_bs;

    // zero super-block of every plane (never overwritten by the x staging)
    for (int i = threadIdx.x; i < 4 * NP; i += nthr)
#pragma unroll
        for (int sp = 0; sp < NSPLIT; ++sp) xs[(size_t)sp * plane + (size_t)M * xrow + i] = 0u;

    const int per_sb = NGS * M;
    const int SPB = max(1, (8 * NPASS) / per_sb);
    const int nslots = SPB * per_sb;
    const int gmul = G < SB ? __ffs(SB / G) - 1 : 0;
    const int gdiv = G > SB ? __ffs(G / SB) - 1 : 0;
    const int useg = (t * UC) / segsz;
    int bsbi[NPASS], brow[NPASS];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp) {
        const int j = 8 * pp + g;
        const int m = j % M, q = j / M, gs = q % NGS, sbi = q / NGS;
        bsbi[pp] = (j < nslots && gs == useg) ? sbi : -1;
        brow[pp] = m;
    }
    int dsbi[NPASS][2], dgs[NPASS][2], dm[NPASS][2];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int j = 8 * pp + 2 * t + c;
            const int q = j / M;
            dm[pp][c] = j % M;
            dgs[pp][c] = q % NGS;
            dsbi[pp][c] = j < nslots ? q / NGS : -1;
        }

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

        float D[NPASS][4], Y[NPASS][4], sc[NPASS][4], bi[NPASS][4];
#pragma unroll
        for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
            for (int e = 0; e < 4; ++e) { D[pp][e] = 0.f; Y[pp][e] = 0.f; sc[pp][e] = 0.f; bi[pp][e] = 0.f; }

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
                    sx[(size_t)m * NSEG + sg] = a;
                    sxt[(size_t)m * NSEG + sg] = b;
                }
                consumer_sync(nthr);
                x_whole = (TSB >= NSBK);
            }

            // ---- this warp's super-blocks of the tile, stage by stage -------
            const int end = t0 + tn;
            int sb = t0 + wkid;
            int bi_ = 0;
            for (int ks = t0 / S; ks * S < end; ++ks) {
                const int slot = it % STAGES, f = it / STAGES;
                if (ok && !mbar_wait(full(slot), (uint32_t)(f & 1))) {
                    ok = false;
                    if (lane == 0) atomicOr(p.fault, 1u);
                }
                const int send = min(end, (ks + 1) * S);
                if (ok) {
                    const unsigned char* st = ring + (size_t)slot * stage_bytes + (size_t)(wrid * 16 + g) * pitch + t * UB;
                    for (; sb < send; sb += wk) {
                        uint32_t wg[NW], wh[NW];
                        const unsigned char* u = st + (sb - ks * S) * 4 * UB;
                        if constexpr (UB == 16) {
                            const uint4 a = *reinterpret_cast<const uint4*>(u);
                            const uint4 b = *reinterpret_cast<const uint4*>(u + 8 * pitch);
                            wg[0] = a.x; wg[1] = a.y; wg[2] = a.z; wg[3] = a.w;
                            wh[0] = b.x; wh[1] = b.y; wh[2] = b.z; wh[3] = b.w;
                        } else {
#pragma unroll
                            for (int q = 0; q < NW; ++q) {
                                wg[q] = reinterpret_cast<const uint32_t*>(u)[q];
                                wh[q] = reinterpret_cast<const uint32_t*>(u + 8 * pitch)[q];
                            }
                        }
                        if (bi_ == 0) {
                            // new batch: scales / biases of its slots (used at batch end)
#pragma unroll
                            for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int c = e & 1;
                                    const int sbs = sb + dsbi[pp][c] * wk;
                                    sc[pp][e] = 0.f; bi[pp][e] = 0.f;
                                    if (dsbi[pp][c] >= 0 && sbs < end) {
                                        const int grp = ((sbs << gmul) >> gdiv) + dgs[pp][c];
                                        sc[pp][e] = DT<T>::ld((e >> 1) ? sch : scg, grp);
                                        bi[pp][e] = DT<T>::ld((e >> 1) ? bih : big, grp);
                                    }
                                }
                        }
                        int xoff[NPASS];
#pragma unroll
                        for (int pp = 0; pp < NPASS; ++pp)
                            xoff[pp] = bsbi[pp] == bi_ ? brow[pp] * xrow + ((sb - t0) * 4 + t) * NP
                                                       : M * xrow + t * NP;
                        tc_steps<B, NPASS, NSPLIT>(std::make_integer_sequence<int, NSTEP / 2>{}, wg, wh, D, xs, xoff,
                                                   plane);
                        if (bi_ == SPB - 1 || sb + wk >= end) {
                            const int sb_first = sb - bi_ * wk;
#pragma unroll
                            for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int c = e & 1;
                                    float a = 0.f, b = 0.f;
                                    if (dsbi[pp][c] >= 0 && dsbi[pp][c] <= bi_) {
                                        const int sl = (sb_first + dsbi[pp][c] * wk - t0) * NGS + dgs[pp][c];
                                        a = sx[(size_t)dm[pp][c] * NSEG + sl];
                                        b = sxt[(size_t)dm[pp][c] * NSEG + sl];
                                    }
                                    Y[pp][e] = fmaf(sc[pp][e], fmaf(-128.f, b, D[pp][e]), fmaf(bi[pp][e], a, Y[pp][e]));
                                    D[pp][e] = 0.f;
                                }
                            bi_ = 0;
                        } else {
                            ++bi_;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(slot));
                ++it;
            }
        }

        if (rb + (int)gridDim.x >= nrb) grid_launch_dependents();

        // ---- reduce over slots of the same x row and over k-warps, store -----
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
