// la_prefill_tc.cu -- chunkwise causal linear-attention prefill on the B200
// tensor cores (sm_100a: TMA + tcgen05 + TMEM).
//
// The computation is the chunkwise form of the slides "Chunking, causality,
// and parallel prefill" (sections "Split into chunks", "Causal triangle",
// "Incoming and outgoing state"): for every chunk c of C tokens of a unit,
//     A   = Q_c K_c^T                      (C x C, fp32 in TMEM)
//     P   = A with j > i set to 0          (diagonal kept; bf16 in smem)
//     O_c = Q_c S_{c-1} + P V_c            (one fp32 TMEM accumulator)
//     S_c = S_{c-1} + K_c^T V_c            (fp32 in TMEM for the whole unit)
// The only serial hop between chunks is S: after K_c^T V_c lands in TMEM,
// the state is copied out once as a bf16 operand for the next chunk's Q S.
//
// One persistent CTA per SM walks units (one sequence of one head) with a
// static stride.  Warp roles (512 threads):
//   warp 0       TMA producer: Q/K/V chunk tiles into an NS-deep ring
//   warps 1-3    MMA issuers (one thread each: output, state, scores);
//                warp 1 also owns the TMEM allocation
//   warps 4-7    "mask" warpgroup: scores -> causal mask -> bf16 P
//   warps 8-11   "state" warpgroup: S_0 in, state hop S -> bf16 operand, S_T out
//   warps 12-15  "output" warpgroup: O TMEM -> bf16 -> smem -> TMA store
// The mask and the state hop run in different warpgroups so that the two
// per-chunk chains (scores -> P -> P V, and S -> bf16 S -> next Q S) overlap.
// Every wait is an mbarrier wait bounded by a timeout; on expiry the kernel
// records the error word, every role winds down, outstanding copies and
// MMAs are drained (bounded), TMEM is freed and the kernel returns.
#include "la_device.cuh"
#include "la_internal.h"

namespace la {

// Optional event trace (compiled in only with -DLINATTN_TRACE): CTA 0 stores
// the SM clock of event `ev` of chunk `g` at trace[ev * (cap / 64) + g]
// (plain stores: no atomics on the traced threads).
#ifdef LINATTN_TRACE
#define LA_TRACE(ev, g)                                                                         \
    do {                                                                                        \
        if (p.trace && blockIdx.x == 0 && (g) < static_cast<int64_t>(p.trace_cap / 64))          \
            p.trace[(ev) * (p.trace_cap / 64) + (g)] = clock64();                               \
    } while (0)
#else
#define LA_TRACE(ev, g) \
    do {                \
    } while (0)
#endif

template <int C, int D>
struct TcCfg {
    static constexpr int kThreads = 512;
    // Rows of the attention MMAs (Q K^T, Q S, P V).  tcgen05 has no M below
    // 64, so a chunk of 16 or 32 tokens runs M = 64 tiles whose first C rows
    // are the chunk; the other rows of the Q and P tiles are zero and their
    // accumulator rows are never read.
    static constexpr int MR = C < 64 ? 64 : C;
    static constexpr int PANEL = C * 128;   // one 64-column panel of a K/V/O chunk tile (bytes)
    static constexpr int QPANEL = MR * 128; // one panel of the Q tile (padded to MR rows)
    static constexpr int NPAN = D / 64;
    static constexpr int TILE = C * D * 2;
    static constexpr int QTILE = MR * D * 2;
    static constexpr int STAGE = QTILE + 2 * TILE;  // Q, K, V of one chunk
    static constexpr int STAGE_TX = 3 * TILE;       // bytes the TMA writes into a stage
    // C = 128: P stays in tensor memory (written over the fp32 scores it came
    // from, read by the P V MMA straight from TMEM) and O is staged for its
    // TMA store in the chunk's own Q tile, which is dead by then; the shared
    // memory this frees buys a deeper Q/K/V ring.  C <= 64 (M = 64 tiles) keeps
    // P and the O staging in their own shared-memory buffers.
    static constexpr bool PT = (C == 128);
    static constexpr int PB = PT ? 0 : 2;                       // P buffers in smem
    static constexpr int OB = (C == 128 && D == 128) ? 1 : 2;  // O accumulators in TMEM
    static constexpr int OSB = PT ? 0 : 2;                      // O staging buffers in smem
    static constexpr int PK = C < 64 ? 64 : C;                  // P row width (keys, padded)
    static constexpr int P_BYTES = MR * PK * 2;
    static constexpr int P_PANEL = MR * 128;
    static constexpr int SB_BYTES = D * D * 2;
    static constexpr int SB_PANEL = D * 128;
    static constexpr int OST_BYTES = C * D * 2;
    static constexpr int NBAR = 80;
    static constexpr int kRing = 16;  // work-item ring (dynamic walk)
    static constexpr int FIXED = PB * P_BYTES + SB_BYTES + OSB * OST_BYTES + NBAR * 8 + 16 + 1024;
    // ring depth: C = 128 and C = 64 as tuned; smaller chunks as deep as fits (<= 8)
    static constexpr int NS_FIT = (232448 - FIXED) / STAGE;
    static constexpr int NS = PT ? (D == 128 ? 2 : 4)
                                 : (C == 64 ? (D == 64 ? 6 : 3) : (NS_FIT < 8 ? NS_FIT : 8));
    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_P = OFF_STAGE + NS * STAGE;
    static constexpr int OFF_SB = OFF_P + PB * P_BYTES;
    static constexpr int OFF_OST = OFF_SB + SB_BYTES;
    static constexpr int OFF_BAR = OFF_OST + OSB * OST_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_RING = OFF_MISC + 16;
    static constexpr int SMEM = OFF_RING + kRing * 8 + 1024;  // + slack to align the base to 1 KB
    // tensor memory columns (fp32, 128 lanes)
    static constexpr int TM_S = 0;
    static constexpr int TM_O = D;
    static constexpr int TM_A = D + OB * D;
    static constexpr int TM_COLS = 512;
    static constexpr int A_COLS = C < 64 ? 64 : C;  // columns per score buffer (64-aligned)
    static_assert(C % 16 == 0 && C >= 16 && C <= 128, "chunk size");
    static_assert(TM_A + 2 * A_COLS <= TM_COLS, "tensor memory budget");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(NS >= 2 && NS <= 8, "barrier slots");
    // mbarrier slots
    static constexpr int B_FULL = 0;       // [NS] TMA landed
    static constexpr int B_EMPTY = 8;      // [NS] MMAs of the stage done
    static constexpr int B_AFULL = 16;     // [2] scores in TMEM
    static constexpr int B_AEMPTY = 18;    // [2] scores read out
    static constexpr int B_PFULL = 20;     // [2] P written
    static constexpr int B_PEMPTY = 22;    // [2] P consumed
    static constexpr int B_SFULL = 24;     // state accumulated
    static constexpr int B_SREAD = 25;     // state read out (may accumulate again)
    static constexpr int B_SBFULL = 26;    // bf16 state operand written
    static constexpr int B_SBEMPTY = 27;   // bf16 state operand consumed
    static constexpr int B_OFULL = 28;     // [2] O accumulated
    static constexpr int B_OEMPTY = 30;    // [2] O read out
    static constexpr int B_OSTFULL = 32;   // [2] O staging written
    static constexpr int B_OSTFREE = 34;   // [2] O staging read by the TMA store
    static constexpr int B_MMADONE = 36;   // [3] drain at teardown (one per issuing thread)
    static constexpr int B_ZERO = 40;      // [NS] rows past the sequence end zeroed in K, V
    static constexpr int B_UFULL = 48;     // [kRing] work item published (dynamic walk)
    static constexpr int B_UEMPTY = 64;    // [kRing] work item taken by every consumer warp
    static constexpr int kTakers = 15;     // warps 1..15 take every item
};

struct Unit {
    int group;     // TMA group coordinate (b*H + h dense, h packed)
    int row0;      // first row of this work item
    int len;       // rows of this work item
    int64_t unit;  // state index
    int seg;       // segment of the unit (0 without a split)
    bool last;     // the item that writes S_T
};

// Work item i.  Without a split an item is a unit.  A packed sequence whose
// offsets are out of range or decreasing is treated as empty (its state is
// left untouched).
__device__ __forceinline__ Unit get_unit(const PrefillProblem& p, int64_t i) {
    if (p.cu == nullptr) {
        const int64_t u = i / p.seg_count;
        const int seg = static_cast<int>(i % p.seg_count);
        const int64_t r0 = seg * p.seg_len;
        const int64_t r1 = min(r0 + p.seg_len, p.rows_per_group);
        return {static_cast<int>(u), static_cast<int>(r0), static_cast<int>(r1 - r0), u, seg,
                seg == p.seg_count - 1};
    }
    // item i: head i % H of the sequence of rank i / H (in the length order
    // when there is one)
    const int n = p.order != nullptr ? p.order[i / p.H] : static_cast<int>(i / p.H);
    const int h = static_cast<int>(i % p.H);
    const int a = p.cu[n];
    const int b = p.cu[n + 1];
    const int64_t unit = static_cast<int64_t>(n) * p.H + h;
    if (a < 0 || b < a || static_cast<int64_t>(b) > p.rows_per_group) return {h, 0, 0, unit, 0, true};
    return {h, a, b - a, unit, 0, true};
}

// Accumulator row held by lane `lane` of a warp reading its TMEM
// sub-partition `sub` with the 32x32b shape.  M = 128: row = lane index in
// TMEM.  M = 64: rows 16*sub .. 16*sub+15 sit in lanes 0..15 of the
// sub-partition; lanes 16..31 hold no row (-1).
template <int M>
__device__ __forceinline__ int acc_row(int sub, int lane) {
    if (M == 128) return sub * 32 + lane;
    return lane < 16 ? sub * 16 + lane : -1;
}

template <int C, int D>
__global__ void __launch_bounds__(512, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmO, const PrefillProblem p) {
    using Cfg = TcCfg<C, D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t tmo = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(&bar[Cfg::B_FULL + s], 1);
            // released by the state stream's K^T V and by the chunk's last
            // other reader: the P V MMA, or (C = 128) the O stores that reuse
            // the Q tile, one per output warp
            mbar_init(&bar[Cfg::B_EMPTY + s], Cfg::PT ? 5 : 2);
            mbar_init(&bar[Cfg::B_ZERO + s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar[Cfg::B_AFULL + b], 1);
            mbar_init(&bar[Cfg::B_AEMPTY + b], 4);
            mbar_init(&bar[Cfg::B_PFULL + b], 4);
            mbar_init(&bar[Cfg::B_PEMPTY + b], 1);
            mbar_init(&bar[Cfg::B_OFULL + b], 1);
            mbar_init(&bar[Cfg::B_OEMPTY + b], 4);
            mbar_init(&bar[Cfg::B_OSTFULL + b], 4);
            mbar_init(&bar[Cfg::B_OSTFREE + b], 1);
        }
        mbar_init(&bar[Cfg::B_SFULL], 1);
        mbar_init(&bar[Cfg::B_SREAD], 4);
        mbar_init(&bar[Cfg::B_SBFULL], 4);
        mbar_init(&bar[Cfg::B_SBEMPTY], 1);
        for (int r = 0; r < Cfg::kRing; ++r) {
            mbar_init(&bar[Cfg::B_UFULL + r], 1);
            mbar_init(&bar[Cfg::B_UEMPTY + r], Cfg::kTakers);
        }
        for (int i = 0; i < 3; ++i) mbar_init(&bar[Cfg::B_MMADONE + i], 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, Cfg::TM_COLS);
        tmem_relinquish();
    }
    if constexpr (Cfg::MR > C) {
        // Pad rows C..MR-1 of every Q panel and of the P tiles: zero once,
        // never written again (the TMA fills rows 0..C-1 only).
        constexpr int kPad = (Cfg::MR - C) * 128 / 16;  // 16-byte pieces per panel
        const uint32_t sb = smem_u32(smem);
        for (int i = threadIdx.x; i < (Cfg::NS * Cfg::NPAN + Cfg::PB) * kPad; i += blockDim.x) {
            const int t = i / kPad, r = i % kPad;
            const uint32_t panel = t < Cfg::NS * Cfg::NPAN
                                       ? Cfg::OFF_STAGE + (t / Cfg::NPAN) * Cfg::STAGE + (t % Cfg::NPAN) * Cfg::QPANEL
                                       : Cfg::OFF_P + (t - Cfg::NS * Cfg::NPAN) * Cfg::P_BYTES;
            st_shared_v4(sb + panel + C * 128 + r * 16, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;
    // Launched as a programmatic dependent of the previous kernel (unsplit
    // input): the set-up above overlapped its tail; no global memory is
    // touched before this wait (which returns at once for an ordinary launch).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
#ifdef LINATTN_TRACE
    if (p.trace && threadIdx.x == 0 && blockIdx.x < p.trace_cap / 64) {
        p.trace[62 * (p.trace_cap / 64) + blockIdx.x] = globaltimer_ns();
        unsigned int smid;
        asm volatile("mov.u32 %0, %smid;" : "=r"(smid));
        p.trace[61 * (p.trace_cap / 64) + blockIdx.x] = smid;
    }
#endif

    const uint32_t sbase = smem_u32(smem);
    auto stage_q = [&](int s) { return sbase + Cfg::OFF_STAGE + s * Cfg::STAGE; };
    auto stage_k = [&](int s) { return sbase + Cfg::OFF_STAGE + s * Cfg::STAGE + Cfg::QTILE; };
    auto stage_v = [&](int s) { return sbase + Cfg::OFF_STAGE + s * Cfg::STAGE + Cfg::QTILE + Cfg::TILE; };
    // ---- work walk.  Static: item blockIdx.x + k * gridDim.x.  Dynamic (a
    // work counter given): the producer claims items from the global counter
    // and publishes them, in order, in a ring of kRing slots; warps 1..15 take
    // every item from the ring.  Either way the k-th item of the walk is the
    // same for every role; -1 ends the walk, -2 means a wait gave up.
    const int64_t n_items = p.n_units * p.seg_count;
    const bool dyn = p.work_counter != nullptr;
    volatile int64_t* ring = reinterpret_cast<volatile int64_t*>(smem + Cfg::OFF_RING);
    auto item_static = [&](int64_t k) -> int64_t {
        const int64_t i = blockIdx.x + k * static_cast<int64_t>(gridDim.x);
        return i < n_items ? i : -1;
    };
    auto publish_item = [&](int64_t k) -> int64_t {  // producer thread only
        if (!dyn) return item_static(k);
        const int r = static_cast<int>(k % Cfg::kRing);
        if (k >= Cfg::kRing &&
            !mbar_wait(&bar[Cfg::B_UEMPTY + r], ((k / Cfg::kRing) + 1) & 1, abort_flag, tmo, 0x140))
            return -2;
        int64_t i = static_cast<int64_t>(atomicAdd(p.work_counter, 1u));
        if (i >= n_items) i = -1;
        ring[r] = i;
        mbar_arrive(&bar[Cfg::B_UFULL + r]);
        return i;
    };
    auto take_item = [&](int64_t k) -> int64_t {  // whole warp
        if (!dyn) return item_static(k);
        const int r = static_cast<int>(k % Cfg::kRing);
        if (!mbar_wait_warp(&bar[Cfg::B_UFULL + r], (k / Cfg::kRing) & 1, abort_flag, tmo, 0x148)) return -2;
        const int64_t i = ring[r];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[Cfg::B_UEMPTY + r]);
        return i;
    };

    const uint32_t p_base = sbase + Cfg::OFF_P;
    const uint32_t sb_base = sbase + Cfg::OFF_SB;
    const uint32_t ost_base = sbase + Cfg::OFF_OST;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int64_t g = 0;
            int64_t last_g[Cfg::NS];
            for (int s = 0; s < Cfg::NS; ++s) last_g[s] = -1;
            bool ok = true;
            for (int64_t kk = 0; ok; ++kk) {
                const int64_t u = publish_item(kk);
                if (u < 0) {
                    ok = (u == -1);
                    break;
                }
                const Unit un = get_unit(p, u);
                const int nch = (un.len + C - 1) / C;
                for (int c = 0; c < nch; ++c, ++g) {
                    const int s = static_cast<int>(g % Cfg::NS);
                    if (g >= Cfg::NS) {
                        if (!mbar_wait(&bar[Cfg::B_EMPTY + s], ((g / Cfg::NS) + 1) & 1, abort_flag,
                                       tmo, 0x100 + s)) {
                            ok = false;
                            break;
                        }
                    }
                    mbar_arrive_expect_tx(&bar[Cfg::B_FULL + s], Cfg::STAGE_TX);
                    const int row = un.row0 + c * C;
#pragma unroll
                    for (int pn = 0; pn < Cfg::NPAN; ++pn) {
                        tma_load_3d(reinterpret_cast<void*>(smem + (stage_q(s) - sbase) + pn * Cfg::QPANEL),
                                    &tmQ, &bar[Cfg::B_FULL + s], pn * 64, row, un.group);
                        tma_load_3d(reinterpret_cast<void*>(smem + (stage_k(s) - sbase) + pn * Cfg::PANEL),
                                    &tmK, &bar[Cfg::B_FULL + s], pn * 64, row, un.group);
                        tma_load_3d(reinterpret_cast<void*>(smem + (stage_v(s) - sbase) + pn * Cfg::PANEL),
                                    &tmV, &bar[Cfg::B_FULL + s], pn * 64, row, un.group);
                    }
                    last_g[s] = g;
                    LA_TRACE(1, g);
                    // L2 prefetch of the chunk kPrefetch ahead (same work item):
                    // its shared-memory load then waits on L2, not on HBM.
                    if (p.prefetch > 0 && c + p.prefetch < nch) {
                        const int prow = un.row0 + (c + p.prefetch) * C;
#pragma unroll
                        for (int pn = 0; pn < Cfg::NPAN; ++pn) {
                            tma_prefetch_l2_3d(&tmQ, pn * 64, prow, un.group);
                            tma_prefetch_l2_3d(&tmK, pn * 64, prow, un.group);
                            tma_prefetch_l2_3d(&tmV, pn * 64, prow, un.group);
                        }
                    }
                }
            }
            if (!ok || *abort_flag) {
                // Let every copy this thread started land before the CTA exits.
                for (int s = 0; s < Cfg::NS; ++s)
                    if (last_g[s] >= 0)
                        mbar_wait_drain(&bar[Cfg::B_FULL + s], (last_g[s] / Cfg::NS) & 1, tmo);
            }
        }
    } else if (warp >= 1 && warp <= 3) {
        // ----------------------------------------------------- MMA issuers
        // Three threads issue tcgen05 MMAs.  An issuing thread blocks while the
        // tensor pipe is busy, so each stream waits only on its own inputs:
        //   warp 3 (scores): A = Q K^T as soon as the chunk's tiles have landed
        //     and its score buffer is free.
        //   warp 1 (output): O = Q S_prev once the bf16 state operand is
        //     written, then O += P V once the mask warpgroup has written P.
        //   warp 2 (state carry): rows past a sequence end are zeroed in K and
        //     V, then S += K^T V as soon as the previous state has been read.
        constexpr uint32_t kIdQK = idesc_bf16_f32(Cfg::MR, C, false, false);
        constexpr uint32_t kIdKV = idesc_bf16_f32(D, D, true, true);
        constexpr uint32_t kIdQS = idesc_bf16_f32(Cfg::MR, D, false, true);
        constexpr uint32_t kIdPV = idesc_bf16_f32(Cfg::MR, D, false, true);
        bool ok = true;
        bool issued_any = false;
        // (unit, chunk) walk
        struct Cursor {
            int64_t u;   // work item
            int64_t kk;  // items taken so far
            int c, nch, nv;
            int64_t g;
            bool valid;
        };
        auto next_nonempty = [&](Cursor& k) {  // next item with at least one chunk
            for (;;) {
                const int64_t u = take_item(k.kk++);
                if (u < 0) {
                    k.valid = false;
                    if (u == -2) ok = false;
                    return;
                }
                const Unit un = get_unit(p, u);
                const int nch = (un.len + C - 1) / C;
                if (nch > 0) {
                    k.u = u;
                    k.c = 0;
                    k.nch = nch;
                    k.nv = min(C, un.len);
                    k.valid = true;
                    return;
                }
            }
        };
        auto first = [&](Cursor& k) {
            k.g = 0;
            k.kk = 0;
            next_nonempty(k);
        };
        auto advance = [&](Cursor& k) {
            ++k.g;
            if (++k.c < k.nch) {
                const Unit un = get_unit(p, k.u);
                k.nv = min(C, un.len - k.c * C);
                return;
            }
            next_nonempty(k);
        };

        if (warp == 2) {
            // ------------------------------------------------ state stream
            const uint32_t tm_S = tmem + Cfg::TM_S;
            Cursor k;
            for (first(k); ok && k.valid; advance(k)) {
                const int64_t g = k.g;
                const int s = static_cast<int>(g % Cfg::NS);
                if (!mbar_wait_warp(&bar[Cfg::B_FULL + s], (g / Cfg::NS) & 1, abort_flag, tmo, 0x200 + s)) {
                    ok = false;
                    break;
                }
                if (k.nv < C) {
                    // Rows past the end of the sequence must not reach the
                    // state (nor, through P = 0 on them, the output).
                    const int nrow = C - k.nv;
                    const int per_tile = nrow * Cfg::NPAN * 8;  // 16-byte pieces
                    for (int i = lane; i < 2 * per_tile; i += 32) {
                        const int t = i / per_tile;
                        const int r = i % per_tile;
                        const int row = k.nv + r / (Cfg::NPAN * 8);
                        const int pn = (r / 8) % Cfg::NPAN;
                        const int ch = r % 8;
                        const uint32_t base = t == 0 ? stage_k(s) : stage_v(s);
                        st_shared_v4(base + pn * Cfg::PANEL + row * 128 + ch * 16, 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                int okw = 1;
                if (lane == 0) {
                    mbar_arrive(&bar[Cfg::B_ZERO + s]);
                    if (!mbar_wait(&bar[Cfg::B_SREAD], g & 1, abort_flag, tmo, 0x220)) okw = 0;
                    LA_TRACE(4, g);
                    if (okw) {
                        tc_fence_after();
                        const uint32_t kb = stage_k(s), vb = stage_v(s);
#pragma unroll
                        for (int ks = 0; ks < C / 16; ++ks)
                            mma_bf16_ss(tm_S, sdesc_sw128(kb + ks * 2048, Cfg::PANEL, 1024),
                                        sdesc_sw128(vb + ks * 2048, Cfg::PANEL, 1024), kIdKV, 1);
                        mma_commit(&bar[Cfg::B_SFULL]);
                        mma_commit(&bar[Cfg::B_EMPTY + s]);
                        issued_any = true;
                    }
                }
                ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
            }
        } else if (warp == 3) {
            // ----------------------------------------------- scores stream
            Cursor k;
            for (first(k); ok && k.valid; advance(k)) {
                const int64_t g = k.g;
                const int s = static_cast<int>(g % Cfg::NS);
                const int b = static_cast<int>(g & 1);
                if (!mbar_wait_warp(&bar[Cfg::B_FULL + s], (g / Cfg::NS) & 1, abort_flag, tmo, 0x208 + s)) {
                    ok = false;
                    break;
                }
                if (lane == 0) LA_TRACE(2, g);
                int okw = 1;
                if (lane == 0) {
                    // buffer b was last used by chunk g-2: its scores have been
                    // read, and (P in TMEM) its P V has completed
                    if (g >= 2 &&
                        !mbar_wait(&bar[Cfg::B_AEMPTY + b], ((g >> 1) + 1) & 1, abort_flag, tmo, 0x210 + b))
                        okw = 0;
                    if (Cfg::PT && okw && g >= 2 &&
                        !mbar_wait(&bar[Cfg::B_PEMPTY + b], ((g >> 1) + 1) & 1, abort_flag, tmo, 0x218 + b))
                        okw = 0;
                    if (okw) {
                        tc_fence_after();
                        const uint32_t tm_A = tmem + Cfg::TM_A + b * Cfg::A_COLS;
                        const uint32_t qb = stage_q(s), kb = stage_k(s);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t qoff = (ks >> 2) * Cfg::QPANEL + (ks & 3) * 32;
                            const uint32_t koff = (ks >> 2) * Cfg::PANEL + (ks & 3) * 32;
                            mma_bf16_ss(tm_A, sdesc_sw128(qb + qoff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                                        kIdQK, ks > 0);
                        }
                        mma_commit(&bar[Cfg::B_AFULL + b]);
                        issued_any = true;
                        LA_TRACE(3, g);
                    }
                }
                ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
            }
        } else {
            // ----------------------------------------------- output stream
            Cursor k;
            for (first(k); ok && k.valid; advance(k)) {
                const int64_t g = k.g;
                const int s = static_cast<int>(g % Cfg::NS);
                const int b = static_cast<int>(g & 1);
                const int ob = static_cast<int>(g % Cfg::OB);
                const uint32_t tm_O = tmem + Cfg::TM_O + ob * D;
                if (!mbar_wait_warp(&bar[Cfg::B_FULL + s], (g / Cfg::NS) & 1, abort_flag, tmo, 0x228 + s)) {
                    ok = false;
                    break;
                }
                int okw = 1;
                if (lane == 0) {
                    // O = Q S_prev
                    if (g >= Cfg::OB &&
                        !mbar_wait(&bar[Cfg::B_OEMPTY + ob], ((g / Cfg::OB) + 1) & 1, abort_flag, tmo, 0x230 + ob))
                        okw = 0;
                    if (okw && !mbar_wait(&bar[Cfg::B_SBFULL], g & 1, abort_flag, tmo, 0x240)) okw = 0;
                    LA_TRACE(5, g);
                    if (okw) {
                        tc_fence_after();
                        const uint32_t qb = stage_q(s);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks >> 2) * Cfg::QPANEL + (ks & 3) * 32;
                            mma_bf16_ss(tm_O, sdesc_sw128(qb + off, 16, 1024),
                                        sdesc_sw128(sb_base + ks * 2048, Cfg::SB_PANEL, 1024), kIdQS, ks > 0);
                        }
                        mma_commit(&bar[Cfg::B_SBEMPTY]);
                        issued_any = true;
                    }
                    // O += P V (a partial chunk also waits for its zeroed V rows)
                    if (okw && !mbar_wait(&bar[Cfg::B_PFULL + b], (g >> 1) & 1, abort_flag, tmo, 0x250 + b)) okw = 0;
                    if (okw && k.nv < C &&
                        !mbar_wait(&bar[Cfg::B_ZERO + s], (g / Cfg::NS) & 1, abort_flag, tmo, 0x260 + s))
                        okw = 0;
                    LA_TRACE(6, g);
                    if (okw) {
                        tc_fence_after();
                        const uint32_t vb = stage_v(s);
                        if constexpr (Cfg::PT) {
                            const uint32_t tm_P = tmem + Cfg::TM_A + b * Cfg::A_COLS;  // 8 columns per 16 keys
#pragma unroll
                            for (int ks = 0; ks < C / 16; ++ks)
                                mma_bf16_ts(tm_O, tm_P + ks * 8, sdesc_sw128(vb + ks * 2048, Cfg::PANEL, 1024),
                                            kIdPV, 1);
                            mma_commit(&bar[Cfg::B_PEMPTY + b]);
                            mma_commit(&bar[Cfg::B_OFULL + ob]);
                        } else {
                            const uint32_t pb = p_base + b * Cfg::P_BYTES;
#pragma unroll
                            for (int ks = 0; ks < C / 16; ++ks) {
                                const uint32_t off = (ks >> 2) * Cfg::P_PANEL + (ks & 3) * 32;
                                mma_bf16_ss(tm_O, sdesc_sw128(pb + off, 16, 1024),
                                            sdesc_sw128(vb + ks * 2048, Cfg::PANEL, 1024), kIdPV, 1);
                            }
                            mma_commit(&bar[Cfg::B_PEMPTY + b]);
                            mma_commit(&bar[Cfg::B_OFULL + ob]);
                            mma_commit(&bar[Cfg::B_EMPTY + s]);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
            }
        }
        if (lane == 0 && issued_any) {
            // Drain: every MMA this thread issued has completed before TMEM is freed.
            mma_commit(&bar[Cfg::B_MMADONE + warp - 1]);
            mbar_wait_drain(&bar[Cfg::B_MMADONE + warp - 1], 0, tmo);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ----------------------------------------------------- mask warpgroup
        const int sub = warp & 3;
        const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
        const int rowA0 = acc_row<Cfg::MR>(sub, lane);
        const int rowA = rowA0 < C ? rowA0 : -1;  // score / P row (-1: none, or a pad row)
        int64_t g = 0;
        bool ok = true;
        for (int64_t kk = 0; ok; ++kk) {
            const int64_t u = take_item(kk);
            if (u < 0) {
                ok = (u == -1);
                break;
            }
            const Unit un = get_unit(p, u);
            const int nch = (un.len + C - 1) / C;
            for (int c = 0; c < nch; ++c, ++g) {
                const int b = static_cast<int>(g & 1);
                // P = mask(A)
                if (!mbar_wait_warp(&bar[Cfg::B_AFULL + b], (g >> 1) & 1, abort_flag, tmo, 0x310 + b)) {
                    ok = false;
                    break;
                }
                if (warp == 4 && lane == 0) LA_TRACE(10, g);
                tc_fence_after();
                if (!Cfg::PT && g >= 2 &&
                    !mbar_wait_warp(&bar[Cfg::B_PEMPTY + b], ((g >> 1) + 1) & 1, abort_flag, tmo, 0x320 + b)) {
                    ok = false;
                    break;
                }
                const uint32_t tm_A = tmem + Cfg::TM_A + b * Cfg::A_COLS + lane_off;
                const uint32_t pb = p_base + b * Cfg::P_BYTES;
                if constexpr (Cfg::PT) {
                    // P (bf16 pairs) over the first C/2 columns of the scores:
                    // half h reads score columns [64h, 64h+64) and writes P
                    // columns [32h, 32h+32), all of which it has already read.
#pragma unroll
                    for (int h = 0; h < C / 64; ++h) {
                        uint32_t r0[32], r1[32], w[32];
                        tmem_ld32(tm_A + h * 64, r0);
                        tmem_ld32(tm_A + h * 64 + 32, r1);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int j = h * 64 + 2 * e;
                            w[e] = pack_bf16x2(j <= rowA ? __uint_as_float(r0[2 * e]) : 0.f,
                                               j + 1 <= rowA ? __uint_as_float(r0[2 * e + 1]) : 0.f);
                            const int j2 = j + 32;
                            w[16 + e] = pack_bf16x2(j2 <= rowA ? __uint_as_float(r1[2 * e]) : 0.f,
                                                    j2 + 1 <= rowA ? __uint_as_float(r1[2 * e + 1]) : 0.f);
                        }
                        tmem_st32(tm_A + h * 32, w);
                    }
                    tmem_wait_st();
                } else if constexpr (C == 16) {
                    uint32_t r[16];
                    tmem_ld16(tm_A, r);
                    tmem_wait_ld();
                    if (rowA >= 0) {
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = ch * 8 + 2 * e;
                                const float a0 = (j <= rowA) ? __uint_as_float(r[ch * 8 + 2 * e]) : 0.f;
                                const float a1 = (j + 1 <= rowA) ? __uint_as_float(r[ch * 8 + 2 * e + 1]) : 0.f;
                                w[e] = pack_bf16x2(a0, a1);
                            }
                            st_shared_v4(pb + sw128_off(rowA, ch), w[0], w[1], w[2], w[3]);
                        }
                    }
                } else
#pragma unroll
                for (int cb = 0; cb < C / 32; ++cb) {
                    uint32_t r[32];
                    tmem_ld32(tm_A + cb * 32, r);
                    tmem_wait_ld();
                    if (rowA >= 0) {
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = cb * 32 + ch * 8 + 2 * e;
                                const float a0 = (j <= rowA) ? __uint_as_float(r[ch * 8 + 2 * e]) : 0.f;
                                const float a1 = (j + 1 <= rowA) ? __uint_as_float(r[ch * 8 + 2 * e + 1]) : 0.f;
                                w[e] = pack_bf16x2(a0, a1);
                            }
                            const int col = cb * 32 + ch * 8;
                            st_shared_v4(pb + (col >> 6) * Cfg::P_PANEL + sw128_off(rowA, (col & 63) >> 3),
                                         w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                tc_fence_before();
                if constexpr (!Cfg::PT) fence_proxy_async_smem();  // P went to shared memory
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bar[Cfg::B_AEMPTY + b]);
                    mbar_arrive(&bar[Cfg::B_PFULL + b]);
                    if (warp == 4) LA_TRACE(11, g);
                }
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // ---------------------------------------------------- state warpgroup
        const int sub = warp & 3;
        const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
        const int rowS = acc_row<D>(sub, lane);  // state row (key index)
        const uint32_t tm_S = tmem + Cfg::TM_S + lane_off;
        int64_t g = 0;
        bool ok = true;
        for (int64_t kk = 0; ok; ++kk) {
            const int64_t u = take_item(kk);
            if (u < 0) {
                ok = (u == -1);
                break;
            }
            const Unit un = get_unit(p, u);
            const int nch = (un.len + C - 1) / C;
            if (nch == 0) continue;
            float* st_row = p.state + un.unit * static_cast<int64_t>(D) * D +
                            static_cast<int64_t>(rowS < 0 ? 0 : rowS) * D;
            // a segment after the first starts from its precomputed state
            // (S_0 plus the K^T V sums of everything before it)
            // (with a split every segment, the first included, reads its start
            // state from the workspace: the state buffer itself is written by
            // the last segment and is never read by another work item)
            const float* in_row = p.seg_count > 1 ? p.seg_states +
                                                        (un.unit * static_cast<int64_t>(p.seg_count) + un.seg) * D * D +
                                                        static_cast<int64_t>(rowS < 0 ? 0 : rowS) * D
                                                  : st_row;
            // ---- unit start: S_0 into TMEM (fp32) and into the bf16 operand
            if (g > 0 && !mbar_wait_warp(&bar[Cfg::B_SBEMPTY], (g - 1) & 1, abort_flag, tmo, 0x300)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t r[32];
                if (rowS >= 0) {
                    const float4* src = reinterpret_cast<const float4*>(in_row + cb * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 f = src[i];
                        r[4 * i + 0] = __float_as_uint(f.x);
                        r[4 * i + 1] = __float_as_uint(f.y);
                        r[4 * i + 2] = __float_as_uint(f.z);
                        r[4 * i + 3] = __float_as_uint(f.w);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                }
                tmem_st32(tm_S + cb * 32, r);
                if (rowS >= 0) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int col = cb * 32 + ch * 8;  // 8 bf16 = one 16-byte chunk
                        const uint32_t addr = sb_base + (col >> 6) * Cfg::SB_PANEL +
                                              sw128_off(rowS, (col & 63) >> 3);
                        st_shared_v4(addr,
                                     pack_bf16x2(__uint_as_float(r[ch * 8 + 0]), __uint_as_float(r[ch * 8 + 1])),
                                     pack_bf16x2(__uint_as_float(r[ch * 8 + 2]), __uint_as_float(r[ch * 8 + 3])),
                                     pack_bf16x2(__uint_as_float(r[ch * 8 + 4]), __uint_as_float(r[ch * 8 + 5])),
                                     pack_bf16x2(__uint_as_float(r[ch * 8 + 6]), __uint_as_float(r[ch * 8 + 7])));
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar[Cfg::B_SREAD]);
                mbar_arrive(&bar[Cfg::B_SBFULL]);
            }
            // ---- chunk loop
            for (int c = 0; c < nch; ++c, ++g) {
                const bool last = (c == nch - 1);
                // state hop: S_c out of TMEM
                if (!mbar_wait_warp(&bar[Cfg::B_SFULL], g & 1, abort_flag, tmo, 0x330)) {
                    ok = false;
                    break;
                }
                if (warp == 8 && lane == 0) LA_TRACE(20, g);
                tc_fence_after();
                uint32_t pk[D / 2];
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    uint32_t r[32];
                    tmem_ld32(tm_S + cb * 32, r);
                    tmem_wait_ld();
                    if (last && un.last && rowS >= 0) {
                        float4* dst = reinterpret_cast<float4*>(st_row + cb * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                 __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[cb * 16 + i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                }
                tc_fence_before();
                if (!last) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar[Cfg::B_SREAD]);
                    if (warp == 8 && lane == 0) LA_TRACE(21, g);
                    if (!mbar_wait_warp(&bar[Cfg::B_SBEMPTY], g & 1, abort_flag, tmo, 0x340)) {
                        ok = false;
                        break;
                    }
                    if (warp == 8 && lane == 0) LA_TRACE(22, g);
                    if (rowS >= 0) {
#pragma unroll
                        for (int ch = 0; ch < D / 8; ++ch) {
                            const int col = ch * 8;
                            st_shared_v4(sb_base + (col >> 6) * Cfg::SB_PANEL + sw128_off(rowS, (col & 63) >> 3),
                                         pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar[Cfg::B_SBFULL]);
                    if (warp == 8 && lane == 0) LA_TRACE(23, g);
                }
            }
        }
    } else if (warp >= 12) {
        // ---------------------------------------------------- output warpgroup
        const int sub = warp & 3;
        const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
        const int row0 = acc_row<Cfg::MR>(sub, lane);
        const int row = row0 < C ? row0 : -1;  // O row of this thread (-1: none, or a pad row)
        const bool elected = (warp == 12 && lane == 0);
        uint16_t* obase = static_cast<uint16_t*>(p.o);
        int64_t g = 0, f = 0;
        bool ok = true;
        for (int64_t kk = 0; ok; ++kk) {
            const int64_t u = take_item(kk);
            if (u < 0) {
                ok = (u == -1);
                break;
            }
            const Unit un = get_unit(p, u);
            const int nch = (un.len + C - 1) / C;
            for (int c = 0; c < nch; ++c, ++g) {
                const int ob = static_cast<int>(g % Cfg::OB);
                const int nv = min(C, un.len - c * C);
                if (!mbar_wait_warp(&bar[Cfg::B_OFULL + ob], (g / Cfg::OB) & 1, abort_flag, tmo,
                                    0x400 + ob)) {
                    ok = false;
                    break;
                }
                if (warp == 12 && lane == 0) LA_TRACE(30, g);
                tc_fence_after();
                const uint32_t tm_O = tmem + Cfg::TM_O + ob * D + lane_off;
                const int64_t grow0 = static_cast<int64_t>(un.group) * p.rows_per_group + un.row0 + c * C;
                const int st_s = static_cast<int>(g % Cfg::NS);  // this chunk's Q/K/V stage
                if (nv == C) {
                    // Full chunk: TMEM -> bf16 -> swizzled staging tile -> TMA store.
                    const int osb = static_cast<int>(f & 1);
                    if (!Cfg::PT && f >= Cfg::OSB &&
                        !mbar_wait_warp(&bar[Cfg::B_OSTFREE + osb], ((f / 2) + 1) & 1, abort_flag, tmo,
                                        0x410 + osb)) {
                        ok = false;
                        break;
                    }
                    // C = 128 stages O in the chunk's own Q tile: its last readers
                    // (the Q K^T and Q S MMAs) completed before O did.
                    const uint32_t stg = Cfg::PT ? stage_q(st_s) : ost_base + osb * Cfg::OST_BYTES;
#pragma unroll
                    for (int cb = 0; cb < D / 32; ++cb) {
                        uint32_t r[32];
                        tmem_ld32(tm_O + cb * 32, r);
                        tmem_wait_ld();
                        if (row >= 0) {
#pragma unroll
                            for (int ch = 0; ch < 4; ++ch) {
                                const int col = cb * 32 + ch * 8;
                                st_shared_v4(stg + (col >> 6) * Cfg::PANEL + sw128_off(row, (col & 63) >> 3),
                                             pack_bf16x2(__uint_as_float(r[ch * 8 + 0]), __uint_as_float(r[ch * 8 + 1])),
                                             pack_bf16x2(__uint_as_float(r[ch * 8 + 2]), __uint_as_float(r[ch * 8 + 3])),
                                             pack_bf16x2(__uint_as_float(r[ch * 8 + 4]), __uint_as_float(r[ch * 8 + 5])),
                                             pack_bf16x2(__uint_as_float(r[ch * 8 + 6]), __uint_as_float(r[ch * 8 + 7])));
                            }
                        }
                    }
                    tc_fence_before();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&bar[Cfg::B_OEMPTY + ob]);
                        if (!Cfg::PT) mbar_arrive(&bar[Cfg::B_OSTFULL + osb]);
                        if (warp == 12) LA_TRACE(31, g);
                    }
                    if constexpr (Cfg::PT) {
                        // each warp stores its own 32 rows as soon as they are
                        // staged (the O tensor map's box is 32 rows high here)
                        // and hands its share of the stage back once the
                        // store has read them
                        if (lane == 0) {
#pragma unroll
                            for (int pn = 0; pn < Cfg::NPAN; ++pn)
                                tma_store_3d(&tmO, smem + (stg - sbase) + pn * Cfg::PANEL + sub * 32 * 128, pn * 64,
                                             un.row0 + c * C + sub * 32, un.group);
                            bulk_commit_group();
                            bulk_wait_group_read<0>();
                            mbar_arrive(&bar[Cfg::B_EMPTY + st_s]);
                        }
                    } else if (elected) {
                        if (mbar_wait(&bar[Cfg::B_OSTFULL + osb], (f / 2) & 1, abort_flag, tmo, 0x420 + osb)) {
#pragma unroll
                            for (int pn = 0; pn < Cfg::NPAN; ++pn)
                                tma_store_3d(&tmO, smem + (stg - sbase) + pn * Cfg::PANEL, pn * 64,
                                             un.row0 + c * C, un.group);
                            bulk_commit_group();
                            bulk_wait_group_read<1>();
                            if (f >= 1) mbar_arrive(&bar[Cfg::B_OSTFREE + ((f - 1) & 1)]);
                        }
                    }
                    ++f;
                } else {
                    // Last, partial chunk of a sequence: plain stores of the
                    // valid rows only (the next sequence's rows follow).
                    const bool valid = row >= 0 && row < nv;
                    uint4* dst = reinterpret_cast<uint4*>(obase + (grow0 + (valid ? row : 0)) * D);
#pragma unroll
                    for (int cb = 0; cb < D / 32; ++cb) {
                        uint32_t r[32];
                        tmem_ld32(tm_O + cb * 32, r);
                        tmem_wait_ld();
                        if (valid) {
#pragma unroll
                            for (int ch = 0; ch < 4; ++ch)
                                dst[cb * 4 + ch] = make_uint4(
                                    pack_bf16x2(__uint_as_float(r[ch * 8 + 0]), __uint_as_float(r[ch * 8 + 1])),
                                    pack_bf16x2(__uint_as_float(r[ch * 8 + 2]), __uint_as_float(r[ch * 8 + 3])),
                                    pack_bf16x2(__uint_as_float(r[ch * 8 + 4]), __uint_as_float(r[ch * 8 + 5])),
                                    pack_bf16x2(__uint_as_float(r[ch * 8 + 6]), __uint_as_float(r[ch * 8 + 7])));
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar[Cfg::B_OEMPTY + ob]);
                    if (Cfg::PT && lane == 0) mbar_arrive(&bar[Cfg::B_EMPTY + st_s]);
                }
            }
        }
        if (lane == 0) bulk_wait_group<0>();  // every output warp's stores have landed
    }

    tc_fence_before();
    __syncthreads();
#ifdef LINATTN_TRACE
    if (p.trace && threadIdx.x == 0 && blockIdx.x < p.trace_cap / 64)
        p.trace[63 * (p.trace_cap / 64) + blockIdx.x] = globaltimer_ns();
#endif
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Sub-segment states for the intra-sequence split.  Because the state is a
// plain sum (S_t = S_0 + sum over j <= t of k_j v_j^T), the state a segment
// starts from is S_0 plus the K^T V sums of the segments before it; this
// kernel computes those sums for sub-segments of sub_len rows, on the tensor
// cores, one sub-segment per work item:
//   warp 0      TMA producer (K and V chunk tiles, NS-deep ring)
//   warp 1      MMA issuer: S_j += K_c^T V_c, two TMEM accumulators so the
//               next sub-segment accumulates while the last one is written
//   warps 2-5   epilogue: TMEM -> fp32 rows of sub_states
// Waits are bounded as in the prefill kernel.
// ---------------------------------------------------------------------------
template <int C, int D>
struct KvCfg {
    static constexpr int kThreads = 192;
    static constexpr int PANEL = C * 128;
    static constexpr int NPAN = D / 64;
    static constexpr int TILE = C * D * 2;
    static constexpr int STAGE = 2 * TILE;  // K, V
    static constexpr int NS = C >= 64 ? ((3 * STAGE <= 200 * 1024) ? 3 : 2)
                                      : (200 * 1024 / STAGE < 8 ? 200 * 1024 / STAGE : 8);
    static constexpr int OFF_BAR = NS * STAGE;
    static constexpr int SMEM = OFF_BAR + 32 * 8 + 16 + 1024;
    static constexpr int TM_COLS = (2 * D <= 128) ? 128 : 256;
    static constexpr int B_FULL = 0, B_EMPTY = 8, B_AFULL = 16, B_AEMPTY = 18, B_DONE = 20;
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int C, int D>
__global__ void __launch_bounds__(192, 1)
    subsegment_states_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                             const PrefillProblem p, float* __restrict__ sub_states) {
    using Cfg = KvCfg<C, D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_BAR + 32 * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_BAR + 32 * 8 + 4);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t tmo = p.timeout_ns;
    const int64_t n_items = p.n_units * p.subs_per_unit;
    const int nch = static_cast<int>((p.sub_len + C - 1) / C);

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(&bar[Cfg::B_FULL + s], 1);
            mbar_init(&bar[Cfg::B_EMPTY + s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar[Cfg::B_AFULL + b], 1);
            mbar_init(&bar[Cfg::B_AEMPTY + b], 4);
        }
        mbar_init(&bar[Cfg::B_DONE], 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, Cfg::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;
    const uint32_t sbase = smem_u32(smem);
    // programmatic dependent launch: no global memory before this wait
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            int64_t g = 0;
            int64_t last_g[Cfg::NS];
            for (int s = 0; s < Cfg::NS; ++s) last_g[s] = -1;
            bool ok = true;
            for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const int64_t u = it / p.subs_per_unit;
                const int64_t j = it % p.subs_per_unit;
                for (int c = 0; c < nch; ++c, ++g) {
                    const int s = static_cast<int>(g % Cfg::NS);
                    if (g >= Cfg::NS && !mbar_wait(&bar[Cfg::B_EMPTY + s], ((g / Cfg::NS) + 1) & 1, abort_flag,
                                                   tmo, 0x500 + s)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar[Cfg::B_FULL + s], Cfg::STAGE);
                    const int row = static_cast<int>(j * p.sub_len) + c * C;
#pragma unroll
                    for (int pn = 0; pn < Cfg::NPAN; ++pn) {
                        tma_load_3d(smem + s * Cfg::STAGE + pn * Cfg::PANEL, &tmK, &bar[Cfg::B_FULL + s], pn * 64,
                                    row, static_cast<int>(u));
                        tma_load_3d(smem + s * Cfg::STAGE + Cfg::TILE + pn * Cfg::PANEL, &tmV, &bar[Cfg::B_FULL + s],
                                    pn * 64, row, static_cast<int>(u));
                    }
                    last_g[s] = g;
                }
            }
            if (!ok || *abort_flag) {
                for (int s = 0; s < Cfg::NS; ++s)
                    if (last_g[s] >= 0) mbar_wait_drain(&bar[Cfg::B_FULL + s], (last_g[s] / Cfg::NS) & 1, tmo);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t kIdKV = idesc_bf16_f32(D, D, true, true);
            int64_t g = 0, local = 0;
            bool ok = true, issued = false;
            for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++local) {
                const int b = static_cast<int>(local & 1);
                if (local >= 2 && !mbar_wait(&bar[Cfg::B_AEMPTY + b], ((local >> 1) + 1) & 1, abort_flag, tmo,
                                             0x510 + b)) {
                    ok = false;
                    break;
                }
                const uint32_t tm_S = tmem + b * D;
                for (int c = 0; c < nch; ++c, ++g) {
                    const int s = static_cast<int>(g % Cfg::NS);
                    if (!mbar_wait(&bar[Cfg::B_FULL + s], (g / Cfg::NS) & 1, abort_flag, tmo, 0x520 + s)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t kb = sbase + s * Cfg::STAGE, vb = kb + Cfg::TILE;
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        mma_bf16_ss(tm_S, sdesc_sw128(kb + ks * 2048, Cfg::PANEL, 1024),
                                    sdesc_sw128(vb + ks * 2048, Cfg::PANEL, 1024), kIdKV, (c > 0 || ks > 0) ? 1u : 0u);
                    mma_commit(&bar[Cfg::B_EMPTY + s]);
                    issued = true;
                }
                if (ok) mma_commit(&bar[Cfg::B_AFULL + b]);
            }
            if (issued) {
                mma_commit(&bar[Cfg::B_DONE]);
                mbar_wait_drain(&bar[Cfg::B_DONE], 0, tmo);
            }
        }
        __syncwarp();
    } else {
        // epilogue warps 2..5 cover TMEM sub-partitions 2, 3, 0, 1
        const int sub = warp & 3;
        const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
        const int row = acc_row<D>(sub, lane);
        int64_t local = 0;
        for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x, ++local) {
            const int b = static_cast<int>(local & 1);
            if (!mbar_wait_warp(&bar[Cfg::B_AFULL + b], (local >> 1) & 1, abort_flag, tmo, 0x530 + b)) break;
            tc_fence_after();
            float* dst = sub_states + it * static_cast<int64_t>(D) * D + static_cast<int64_t>(row < 0 ? 0 : row) * D;
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t r[32];
                tmem_ld32(tmem + b * D + lane_off + cb * 32, r);
                tmem_wait_ld();
                if (row >= 0) {
                    float4* d4 = reinterpret_cast<float4*>(dst + cb * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        d4[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[Cfg::B_AEMPTY + b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TM_COLS);
    }
}

template <int C, int D>
static cudaError_t launch_sub_impl(const PrefillProblem& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                   float* sub_states, int num_sms, cudaStream_t s) {
    using Cfg = KvCfg<C, D>;
    auto kern = subsegment_states_kernel<C, D>;
    static PerDeviceOnce attrs;
    cudaError_t e = attrs.run(
        [&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM); });
    if (e != cudaSuccess) return e;
    const int64_t items = p.n_units * p.subs_per_unit;
    const int64_t grid = items < num_sms ? items : num_sms;
    if (grid < 1) return cudaSuccess;
    e = launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(Cfg::kThreads), Cfg::SMEM, s, tk, tv, p, sub_states);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_subsegment_states(const PrefillProblem& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                     float* sub_states, int num_sms, cudaStream_t s) {
    if (p.dk == 64 && p.chunk == 16) return launch_sub_impl<16, 64>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 128 && p.chunk == 16) return launch_sub_impl<16, 128>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 64 && p.chunk == 32) return launch_sub_impl<32, 64>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 128 && p.chunk == 32) return launch_sub_impl<32, 128>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 64 && p.chunk == 64) return launch_sub_impl<64, 64>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 128 && p.chunk == 64) return launch_sub_impl<64, 128>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 64 && p.chunk == 128) return launch_sub_impl<128, 64>(p, tk, tv, sub_states, num_sms, s);
    if (p.dk == 128 && p.chunk == 128) return launch_sub_impl<128, 128>(p, tk, tv, sub_states, num_sms, s);
    return cudaErrorInvalidValue;
}

// seg_states[u][s] = S_0[u] + sum_{j < s*k} sub_states[u][j] for every segment
// s (s = 0 is a copy of S_0): one thread per float4 of a unit's state walks
// the sub-segment sums once, in order.  The loads go out eight at a time (the
// additions stay in order, so the sums are the same).
__global__ void segment_prefix_kernel(const float4* __restrict__ s0, const float4* __restrict__ sub,
                                      float4* __restrict__ seg, int64_t n_units, int d4, int subs_per_seg,
                                      int seg_count) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (i >= n_units * d4) return;
    const int64_t u = i / d4, e = i % d4;
    const int subs = (seg_count - 1) * subs_per_seg;
    float4 acc = s0[u * d4 + e];
    seg[(u * seg_count) * d4 + e] = acc;
    for (int j0 = 0; j0 < subs; j0 += 8) {
        float4 x[8];
#pragma unroll
        for (int t = 0; t < 8; ++t)
            if (j0 + t < subs) x[t] = sub[(u * subs + j0 + t) * d4 + e];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int j = j0 + t;
            if (j < subs) {
                acc.x += x[t].x;
                acc.y += x[t].y;
                acc.z += x[t].z;
                acc.w += x[t].w;
                if ((j + 1) % subs_per_seg == 0) seg[(u * seg_count + (j + 1) / subs_per_seg) * d4 + e] = acc;
            }
        }
    }
}

cudaError_t launch_segment_prefix(const PrefillProblem& p, float* seg_states, cudaStream_t s) {
    const int d4 = p.dk * p.dv / 4;
    const int64_t n = p.n_units * d4;
    if (n <= 0) return cudaSuccess;
    const int threads = 256;
    cudaError_t e = launch_pdl(segment_prefix_kernel, dim3(static_cast<unsigned>((n + threads - 1) / threads)),
                               dim3(threads), 0, s, reinterpret_cast<const float4*>(p.state),
                               reinterpret_cast<const float4*>(p.sub_states), reinterpret_cast<float4*>(seg_states),
                               p.n_units, d4, p.subs_per_seg, p.seg_count);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Rank of every sequence when sorted by decreasing length (ties: lower index
// first): each thread counts the sequences that sort before its own, over a
// copy of all lengths in shared memory.
__global__ void length_order_kernel(const int32_t* __restrict__ cu, int num_seqs, int64_t total_rows,
                                    int32_t* __restrict__ order) {
    __shared__ int32_t len[kMaxOrderedSeqs];
    for (int i = threadIdx.x; i < num_seqs; i += blockDim.x) {
        const int a = cu[i], b = cu[i + 1];
        len[i] = (a < 0 || b < a || static_cast<int64_t>(b) > total_rows) ? 0 : b - a;
    }
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= num_seqs) return;
    const int li = len[i];
    int rank = 0;
    for (int j = 0; j < num_seqs; ++j) {
        const int lj = len[j];
        rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    order[rank] = i;
}

cudaError_t launch_length_order(const int32_t* cu, int num_seqs, int64_t total_rows, int32_t* order,
                                cudaStream_t s) {
    if (num_seqs <= 0 || num_seqs > kMaxOrderedSeqs) return cudaErrorInvalidValue;
    const int threads = 256;
    length_order_kernel<<<(num_seqs + threads - 1) / threads, threads, 0, s>>>(cu, num_seqs, total_rows, order);
    return cudaGetLastError();
}

int prefill_tc_o_box_rows(int chunk) { return chunk == 128 ? 32 : chunk; }

bool prefill_tc_supported(int D, int chunk) {
    return (D == 64 || D == 128) && (chunk == 16 || chunk == 32 || chunk == 64 || chunk == 128);
}

template <int C, int D>
static cudaError_t launch_tc_impl(const PrefillProblem& p, const CUtensorMap& tq,
                                  const CUtensorMap& tk, const CUtensorMap& tv,
                                  const CUtensorMap& to, int num_sms, cudaStream_t s) {
    // A CTA of this kernel holds a whole SM's registers, so CTAs launched
    // early as programmatic dependents would take the SMs from the previous
    // kernel while they wait.  After the split's prefix kernel (many small
    // CTAs still to run) the launch is an ordinary one; the grid-dependency
    // wait in the kernel then returns at once.
    const bool pdl = p.seg_count == 1;
    using Cfg = TcCfg<C, D>;
    auto kern = prefill_tc_kernel<C, D>;
    // Raise the dynamic shared-memory limit once per device (not inside a
    // stream capture: the first launch on a device sets it).
    static PerDeviceOnce attrs;
    cudaError_t e = attrs.run(
        [&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM); });
    if (e != cudaSuccess) return e;
    const int64_t items = p.n_units * p.seg_count;
    int64_t grid = items < num_sms ? items : num_sms;
    if (grid < 1) return cudaSuccess;
    if (pdl) {
        e = launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(Cfg::kThreads), Cfg::SMEM, s, tq, tk, tv, to, p);
        if (e != cudaSuccess) return e;
    } else {
        kern<<<static_cast<unsigned>(grid), Cfg::kThreads, Cfg::SMEM, s>>>(tq, tk, tv, to, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const PrefillProblem& p, const CUtensorMap& tq,
                              const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& to, int num_sms, cudaStream_t s) {
    if (p.dk == 64 && p.chunk == 16) return launch_tc_impl<16, 64>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 128 && p.chunk == 16) return launch_tc_impl<16, 128>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 64 && p.chunk == 32) return launch_tc_impl<32, 64>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 128 && p.chunk == 32) return launch_tc_impl<32, 128>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 64 && p.chunk == 64) return launch_tc_impl<64, 64>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 128 && p.chunk == 64) return launch_tc_impl<64, 128>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 64 && p.chunk == 128) return launch_tc_impl<128, 64>(p, tq, tk, tv, to, num_sms, s);
    if (p.dk == 128 && p.chunk == 128) return launch_tc_impl<128, 128>(p, tq, tk, tv, to, num_sms, s);
    return cudaErrorInvalidValue;
}

}  // namespace la
