// vc_attn.cu -- ExpCast-FP8 attention forward on sm_100a tensor cores.
//
// Method (chooseai.io news 7051, section "核心方法之二：ExpCast-FP8 换掉 softmax
// 里的指数"): between the two low-bit GEMMs, a log2-domain score z goes
// straight to an E4M3 probability byte round(8z + 56 + beta) with one FMA, so
// no FP32 exponential and no format conversion sit between the GEMMs.
// V-Smooth's block means return through the per-tile row sums of the online
// softmax (same page, V-Smooth section; theclarity.today: restored during the
// online softmax, one pass over the values).
//
// One CTA computes a 128-row query tile of one (b, h) against all T key tiles
// (the block-sparse instantiation: against the tiles its mask row keeps).
// The A operands of every MMA live in tensor memory, so shared memory only
// feeds the B operands (K tile, V^T tile, a constant tile of ones):
//   TMEM (columns): S0, S1 [BK each] | O [D + 16] | Q [D/4] | P0, P1 [BK/4 each]
//                   (E4M3 A operands: 4 values a column).  O's column D
//                   accumulates the running row sum l: the PV B operand is the
//                   V^T tile followed by 16 rows of E4M3 ones.
//   warp 0      TMA producer: K tile, V^T tile and block mean per key tile
//               through a STAGES-deep ring.
//   warp 1      TMEM owner and MMA issuer (one elected lane), kind::f8f6f4:
//                 S[t%2] = Q K_t^T     (A = Q in TMEM)
//                 [O|l] += P_t [V_t|1] (A = P_t in TMEM; N = D + 16)
//   warps 2..5  softmax, one warp per TMEM lane quadrant, a thread per query
//               row: it first writes the row's E4M3 Q into TMEM; per tile: row
//               max of S, integer row reference M (raised online; a rise by k
//               rescales O by 2^-k, exactly, once PV(t-1) has landed), ExpCast
//               bytes stored to TMEM as the A operand of the PV MMA.
//   warps 6..9  correction, one warp per quadrant: after PV(t), the tile's
//               row sum l_t = l(t) - 2^-k l(t-1) from O's column D; l(t) scaled
//               by the next tile's 2^-k before that tile's PV (both signal
//               p_full with the softmax warps); acc += l_t * mu_t (the
//               block-mean restore), rescaled with O; epilogue
//               O = (v_scale * O + acc) / l in bf16, original token order.
// Every wait is bounded (DevCtl); on a timeout the CTA drains its copies and
// MMAs, frees TMEM and exits with the status word set.  A CTA does nothing
// when the status word already holds an error.
#include "vc_launch.cuh"

namespace vc {

template <int D, int BK>
struct AttnCfg {
    static constexpr int BM = 128;
    static constexpr int STAGES = 4;
    static constexpr int THREADS = 320;  // 10 warps
    static constexpr int K_BYTES = BK * D;
    static constexpr int V_BYTES = D * BK;            // the TMA-loaded V^T tile
    static constexpr int VX_BYTES = (D + 16) * BK;    // + 16 rows of ones (the l column)
    static constexpr int MU_BYTES = D * 4;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
    static constexpr int OFF_MU = OFF_V + STAGES * VX_BYTES;
    static constexpr int OFF_KINC = OFF_MU + STAGES * MU_BYTES;
    static constexpr int OFF_BAR = OFF_KINC + 4 * BM * 4;
    // barrier slots
    static constexpr int B_QREADY = 0;
    static constexpr int B_KFULL = 1;
    static constexpr int B_KEMPTY = B_KFULL + STAGES;
    static constexpr int B_VFULL = B_KEMPTY + STAGES;
    static constexpr int B_VEMPTY = B_VFULL + STAGES;
    static constexpr int B_SFULL = B_VEMPTY + STAGES;
    static constexpr int B_PFULL = B_SFULL + 2;
    static constexpr int B_PVDONE = B_PFULL + 2;
    static constexpr int B_KINC = B_PVDONE + 2;
    static constexpr int B_MMADONE = B_KINC + 4;
    static constexpr int NBAR = B_MMADONE + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
    // TMEM columns
    static constexpr int S_COL0 = 0;
    static constexpr int O_COL = 2 * BK;
    static constexpr int L_COL = O_COL + D;  // running row sum l
    static constexpr int Q_COL = O_COL + D + 16;
    static constexpr int P_COL0 = Q_COL + D / 4;
    static constexpr int TMEM_USED = P_COL0 + 2 * (BK / 4);
    static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert((K_BYTES % 1024) == 0 && (VX_BYTES % 1024) == 0, "swizzled tiles stay 1024-byte aligned");
};

// Block-sparse key tiles: the first kept tile at or after `from` in a query
// tile's mask row (T if none); every tile when there is no mask.
__device__ __forceinline__ int next_kept(const uint8_t* row, int from, int T) {
    if (!row) return from;
    while (from < T && row[from] == 0) ++from;
    return from;
}

// Kept tiles of a mask row, counted by one warp with 16-byte loads (bytes
// past T are read only inside the row's 16-byte-aligned span, never past it).
__device__ __forceinline__ int count_kept(const uint8_t* row, int T, int lane) {
    int n = 0;
    for (int t = lane * 16; t < T; t += 32 * 16) {
        if (t + 16 <= T && (reinterpret_cast<uintptr_t>(row + t) & 15u) == 0) {
            const uint4 w = *reinterpret_cast<const uint4*>(row + t);
            n += __popc(__vcmpne4(w.x, 0u)) / 8 + __popc(__vcmpne4(w.y, 0u)) / 8 + __popc(__vcmpne4(w.z, 0u)) / 8 +
                 __popc(__vcmpne4(w.w, 0u)) / 8;
        } else {
            for (int u = t; u < t + 16 && u < T; ++u) n += row[u] != 0;
        }
    }
    return __reduce_add_sync(0xffffffffu, n);
}

// SPARSE: the block-sparse instantiation (a tile mask is read); the dense one
// compiles without any of it.
template <int D, int BK, bool SPARSE>
__global__ void __launch_bounds__(320, 1)
    vc_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const AttnArgs args) {
    using Cfg = AttnCfg<D, BK>;
    constexpr int STAGES = Cfg::STAGES;
    // The prep outputs are undefined after a recorded device error.
    if (ctl_failed(args.ctl.status)) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * Cfg::BM;
    const int bh = blockIdx.y;
    const int N = args.N;
    const int T = args.T;  // key tiles of the head
    // block-sparse: this query tile's row of the mask (null: every tile)
    const uint8_t* mrow = SPARSE ? args.tile_mask + ((size_t)bh * gridDim.x + blockIdx.x) * T : nullptr;

    auto bar = [&](int i) -> uint32_t { return base + Cfg::OFF_BAR + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
    int* kinc_ring = reinterpret_cast<int*>(smem + Cfg::OFF_KINC);

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        mbar_init(bar(Cfg::B_QREADY), 4);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(Cfg::B_KFULL + s), 1);
            mbar_init(bar(Cfg::B_KEMPTY + s), 1);
            mbar_init(bar(Cfg::B_VFULL + s), 1);
            mbar_init(bar(Cfg::B_VEMPTY + s), 1 + 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(Cfg::B_SFULL + i), 1);
            // P(t) posted by the 4 softmax warps, and l(t-1) read (then scaled)
            // by the 4 correction warps
            mbar_init(bar(Cfg::B_PFULL + i), 4 + 4);
            mbar_init(bar(Cfg::B_PVDONE + i), 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(bar(Cfg::B_KINC + i), 4);
        mbar_init(bar(Cfg::B_MMADONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    int* ta_slot = reinterpret_cast<int*>(smem + Cfg::OFF_MISC + 8);
    if (SPARSE && warp == 2) {  // the number of key tiles this CTA visits
        const int ta = count_kept(mrow, T, lane);
        if (lane == 0) *ta_slot = ta;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    {  // rows D..D+15 of every V stage: E4M3 1.0, so the PV MMA also sums P
        const uint4 v = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
        constexpr int PER = 16 * BK / 16;  // uint4 per stage
        for (int i = threadIdx.x; i < STAGES * PER; i += Cfg::THREADS)
            reinterpret_cast<uint4*>(smem + Cfg::OFF_V + (i / PER) * Cfg::VX_BYTES + Cfg::V_BYTES)[i % PER] = v;
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const DevCtl ctl = args.ctl;
    // TA tiles are visited; visit i counts barrier phases and ring stages, and
    // loads the i-th kept tile (next_kept walks the mask row to it)
    const int TA = SPARSE ? *ta_slot : T;

    if (warp == 0) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int issued_k = 0, issued_v = 0;
            int cursor = SPARSE ? next_kept(mrow, 0, T) : 0;  // the sparse instantiation walks the mask
            for (int t = 0; t < TA; ++t) {
                const int tile = SPARSE ? cursor : t;
                if constexpr (SPARSE) cursor = next_kept(mrow, cursor + 1, T);
                const int st = t % STAGES;
                const int n = t / STAGES;
                if (n > 0 && !mbar_wait(bar(Cfg::B_KEMPTY + st), (n - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(bar(Cfg::B_KFULL + st), Cfg::K_BYTES);
                tma_load_3d(base + Cfg::OFF_K + st * Cfg::K_BYTES, &tm_k, bar(Cfg::B_KFULL + st), 0, tile * BK, bh);
                issued_k = t + 1;
                if (n > 0 && !mbar_wait(bar(Cfg::B_VEMPTY + st), (n - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(bar(Cfg::B_VFULL + st), Cfg::V_BYTES + Cfg::MU_BYTES);
                tma_load_3d(base + Cfg::OFF_V + st * Cfg::VX_BYTES, &tm_v, bar(Cfg::B_VFULL + st), tile * BK, 0, bh);
                bulk_load(base + Cfg::OFF_MU + st * Cfg::MU_BYTES, args.v_mean + ((size_t)bh * T + tile) * D,
                          Cfg::MU_BYTES, bar(Cfg::B_VFULL + st));
                issued_v = t + 1;
            }
            // Drain: every copy issued has landed before the CTA may exit.  Only
            // the last STAGES tiles of each ring can still be in flight.
            for (int t = issued_k - STAGES < 0 ? 0 : issued_k - STAGES; t < issued_k; ++t)
                drain_wait(bar(Cfg::B_KFULL + t % STAGES), (t / STAGES) & 1, ctl);
            for (int t = issued_v - STAGES < 0 ? 0 : issued_v - STAGES; t < issued_v; ++t)
                drain_wait(bar(Cfg::B_VFULL + t % STAGES), (t / STAGES) & 1, ctl);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        // The whole warp runs the loop (warp-uniform operands); one elected
        // lane issues each MMA and commit.  S buffer (t+2)%2 is free once the
        // softmax has posted P(t): it reads S(t) before it writes P(t), and
        // QK(t+2) is issued after this warp waited for p_full(t).
        const uint32_t id_qk = idesc_e4m3_f32(BK);
        const uint32_t id_pv = idesc_e4m3_f32(D + 16);
        bool ok = warp_wait(bar(Cfg::B_QREADY), 0, ctl, abort_flag);
        auto issue_qk = [&](int t) -> bool {
            const int st = t % STAGES, sb = t & 1;
            if (!warp_wait(bar(Cfg::B_KFULL + st), (t / STAGES) & 1, ctl, abort_flag)) return false;
            tc_fence_after();
            const uint64_t dk = smem_desc(base + Cfg::OFF_K + st * Cfg::K_BYTES, D);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
                mma_f8_ts_warp(tmem + Cfg::S_COL0 + sb * BK, tmem + Cfg::Q_COL + 8 * kk, dk + 2 * kk, id_qk, kk > 0);
            mma_commit_warp(bar(Cfg::B_SFULL + sb));
            mma_commit_warp(bar(Cfg::B_KEMPTY + st));
            return true;
        };
        auto issue_pv = [&](int t) -> bool {
            const int st = t % STAGES, pb = t & 1;
            // p_full(t) also carries the correction warps' read of l(t-1) (PV(t)
            // adds into O's l column) and their wait for V(t): one wait here
            if (!warp_wait(bar(Cfg::B_PFULL + pb), (t >> 1) & 1, ctl, abort_flag)) return false;
            tc_fence_after();
            const uint32_t ap = tmem + Cfg::P_COL0 + pb * (BK / 4);
            const uint64_t dv = smem_desc(base + Cfg::OFF_V + st * Cfg::VX_BYTES, BK);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
                mma_f8_ts_warp(tmem + Cfg::O_COL, ap + 8 * kk, dv + 2 * kk, id_pv, (t > 0 || kk > 0) ? 1u : 0u);
            mma_commit_warp(bar(Cfg::B_PVDONE + pb));
            mma_commit_warp(bar(Cfg::B_VEMPTY + st));
            return true;
        };
        if (ok && TA > 0) ok = issue_qk(0);
        for (int t = 0; ok && t < TA; ++t) {
            if (t + 1 < TA && !issue_qk(t + 1)) break;
            if (!issue_pv(t)) break;
        }
        mma_commit_warp(bar(Cfg::B_MMADONE));
        drain_wait(bar(Cfg::B_MMADONE), 0, ctl);
    } else if (warp < 6) {
        // -------------------------------------------------------- softmax
        // One warp per TMEM lane quadrant: warp w handles rows
        // 32qd..32qd+31 (qd = w % 4), a thread the whole row of BK scores.
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_tmem = tmem + ((uint32_t)(qd * 32) << 16);
        const int qrow = q0 + row;
        {   // the row's E4M3 Q into TMEM (zeros past N)
            uint32_t qw[D / 4];
            const uint4* src = reinterpret_cast<const uint4*>(args.q_fp8 + ((size_t)bh * N + qrow) * D);
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                const uint4 v = qrow < N ? src[i] : make_uint4(0u, 0u, 0u, 0u);
                qw[4 * i + 0] = v.x;
                qw[4 * i + 1] = v.y;
                qw[4 * i + 2] = v.z;
                qw[4 * i + 3] = v.w;
            }
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_st16(lane_tmem + Cfg::Q_COL + 16 * c, qw + 16 * c);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_QREADY));
        }
        const float sqv = qrow < N ? args.sq[(size_t)bh * N + qrow] : 0.0f;
        const float aq = __fmul_rn(args.kappa, sqv);
        const float c0 = 56.0f + (float)args.beta;
        float M = 0.0f;
        int tile_next = SPARSE ? next_kept(mrow, 0, T) : 0;  // the sparse instantiation walks the mask
        float sk_next = TA > 0 ? args.k_scale[(size_t)bh * T + tile_next] : 0.0f;
        for (int t = 0; t < TA; ++t) {
            const int sb = t & 1;
            const int tile = SPARSE ? tile_next : t;
            const float sk = sk_next;
            if (t + 1 < TA) {
                if constexpr (SPARSE) tile_next = next_kept(mrow, tile + 1, T);
                sk_next = args.k_scale[(size_t)bh * T + (SPARSE ? tile_next : t + 1)];
            }
            if (!warp_wait(bar(Cfg::B_SFULL + sb), (t >> 1) & 1, ctl, abort_flag)) break;
            tc_fence_after();
            float s[BK];
#pragma unroll
            for (int c = 0; c < BK / 32; ++c) tmem_ld32(lane_tmem + Cfg::S_COL0 + sb * BK + 32 * c, s + 32 * c);
            tmem_wait_ld();

            const int valid = N - tile * BK;
            if (valid < BK) {
#pragma unroll
                for (int j = 0; j < BK; ++j)
                    if (j >= valid) s[j] = -INFINITY;
            }
            // row max: 8 independent 3-input max chains, then a short tree
            float m8[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) m8[a] = fmaxf(s[2 * a], s[2 * a + 1]);
#pragma unroll
            for (int j = 16; j < BK; j += 16)
#pragma unroll
                for (int a = 0; a < 8; ++a) m8[a] = fmax3(m8[a], s[j + 2 * a], s[j + 2 * a + 1]);
            const float mx =
                fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
            const float A = __fmul_rn(aq, sk);
            const float Mc = ceilf(__fmul_rn(__fmul_rn(A, mx), 0.125f));
            const float Mnew = t == 0 ? Mc : fmaxf(M, Mc);
            const int kinc = t == 0 ? 0 : (int)(Mnew - M);
            M = Mnew;
            const float cbm = (c0 - 8.0f * M) + kMagic;
            // k goes out at once: the correction warps scale l by 2^-k when
            // they read it after PV(t-1)
            kinc_ring[(t & 3) * Cfg::BM + row] = kinc;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_KINC + (t & 3)));
            // P slot sb was last read by the PV MMA of tile t-2.  That MMA has
            // completed: one elected thread issues every MMA and commit, a
            // commit tracks all of that thread's earlier MMAs, and QK(t) --
            // whose commit s_full(t) this warp waited for -- was issued after
            // PV(t-2).
            const uint32_t pcol = lane_tmem + Cfg::P_COL0 + sb * (BK / 4);
#pragma unroll
            for (int c = 0; c < BK / 64; ++c) {  // 64 scores -> 16 words of bytes
                uint32_t pw[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const float* sp = s + 64 * c + 4 * q;
                    pw[q] = expcast4(A, sp[0], sp[1], sp[2], sp[3], cbm);
                }
                if (valid < BK) {
                    // Keys past N carry no weight.  Their scores are -inf, which
                    // codes to 0 only while A > 0: with A = 0 (a zero Q row or
                    // an all-zero K block) the FMA gives 0 * -inf = NaN, so the
                    // bytes are cleared here instead.
#pragma unroll
                    for (int q = 0; q < 16; ++q) pw[q] &= tail_keep_mask(valid - (64 * c + 4 * q));
                }
                tmem_st16(pcol + 16 * c, pw);
            }
            if (t > 0 && __any_sync(0xffffffffu, kinc > 0)) {
                // O holds PV of tiles < t: wait for it, then scale O by 2^-kinc
                // (before this tile's PV, which waits on p_full below; l is
                // scaled by the correction warps).  All of O in one round trip.
                if (!warp_wait(bar(Cfg::B_PVDONE + ((t - 1) & 1)), ((t - 1) >> 1) & 1, ctl, abort_flag)) break;
                tc_fence_after();
                const float f = exp2_neg_int(kinc);
                float o[D];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) tmem_ld32(lane_tmem + Cfg::O_COL + 32 * c, o + 32 * c);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < D; ++i) o[i] *= f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) tmem_st32(lane_tmem + Cfg::O_COL + 32 * c, o + 32 * c);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_PFULL + sb));
        }
    } else {
        // -------------------------------------------------------- correction + epilogue
        // One warp per lane quadrant: warp w owns every output channel of
        // rows 32qd..32qd+31 (qd = w % 4).
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_tmem = tmem + ((uint32_t)(qd * 32) << 16);
        const int qrow = q0 + row;
        float acc[D];
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = 0.0f;
        float l = 0.0f;  // running row sum after the last tile seen
        // k of tile 0 (always 0); each later tile's k is read one iteration
        // early, to scale l before that tile's PV.
        bool ok = TA == 0 || warp_wait(bar(Cfg::B_KINC + 0), 0, ctl, abort_flag);
        ok = ok && (TA == 0 || warp_wait(bar(Cfg::B_VFULL + 0), 0, ctl, abort_flag));
        if (ok && TA > 0 && lane == 0) mbar_arrive(bar(Cfg::B_PFULL + 0));  // V(0) landed; no l to read yet
        int kinc = 0;
        for (int t = 0; ok && t < TA; ++t) {
            const int st = t % STAGES;
            if (!(ok = warp_wait(bar(Cfg::B_PVDONE + (t & 1)), (t >> 1) & 1, ctl, abort_flag))) break;
            tc_fence_after();
            const float lt = tmem_ld1(lane_tmem + Cfg::L_COL);
            tmem_wait_ld();
            const int kt = kinc;  // this tile's k
            if (t + 1 < TA) {
                // l(t) * 2^-k(t+1) into O's l column (exact), before PV(t+1),
                // which waits for these warps on p_full(t+1); the softmax scales
                // the rest of O
                const int tn = t + 1;
                if (!(ok = warp_wait(bar(Cfg::B_KINC + (tn & 3)), (tn >> 2) & 1, ctl, abort_flag))) break;
                kinc = kinc_ring[(tn & 3) * Cfg::BM + row];
                if (__any_sync(0xffffffffu, kinc > 0)) {
                    tmem_st1(lane_tmem + Cfg::L_COL, lt * exp2_neg_int(kinc));
                    tmem_wait_st();
                }
            }
            // V(t+1) landed too before p_full(t+1) (the MMA warp relies on it);
            // V(t), read below, was waited for one iteration earlier
            if (t + 1 < TA &&
                !(ok = warp_wait(bar(Cfg::B_VFULL + (t + 1) % STAGES), ((t + 1) / STAGES) & 1, ctl, abort_flag)))
                break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && t + 1 < TA) mbar_arrive(bar(Cfg::B_PFULL + ((t + 1) & 1)));
            float lb;
            if (kt > 0) {
                const float f = exp2_neg_int(kt);
#pragma unroll
                for (int c = 0; c < D; ++c) acc[c] *= f;
                lb = lt - l * f;
            } else {
                lb = lt - l;
            }
            l = lt;
            const float4* mu = reinterpret_cast<const float4*>(smem + Cfg::OFF_MU + st * Cfg::MU_BYTES);
#pragma unroll
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 m = mu[c4];
                const float2 a01 = ffma2(make_float2(lb, lb), make_float2(m.x, m.y),
                                         make_float2(acc[4 * c4 + 0], acc[4 * c4 + 1]));
                const float2 a23 = ffma2(make_float2(lb, lb), make_float2(m.z, m.w),
                                         make_float2(acc[4 * c4 + 2], acc[4 * c4 + 3]));
                acc[4 * c4 + 0] = a01.x;
                acc[4 * c4 + 1] = a01.y;
                acc[4 * c4 + 2] = a23.x;
                acc[4 * c4 + 3] = a23.y;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_VEMPTY + st));
        }
        if (ok && TA > 0) {
            // The last PV has completed, so O is final.
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float* vsc = args.v_scale + (size_t)bh * D;
            __nv_bfloat16* orow = args.out + ((size_t)bh * N + qrow) * D;
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                float o[16];
                tmem_ld16(lane_tmem + Cfg::O_COL + 16 * c, o);
                tmem_wait_ld();
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int c0i = 16 * c + 2 * i;
                    const float x0 = (vsc[c0i] * o[2 * i] + acc[c0i]) * inv_l;
                    const float x1 = (vsc[c0i + 1] * o[2 * i + 1] + acc[c0i + 1]) * inv_l;
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                    packed[i] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                if (qrow < N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 16 * c);
                    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                }
            }
        } else if (SPARSE && ok && TA == 0 && qrow < N) {  // a block-sparse row with no key tile: 0
            uint4* dst = reinterpret_cast<uint4*>(args.out + ((size_t)bh * N + qrow) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    }

    // ------------------------------------------------------------ teardown
    if (warp >= 2 && warp < 6) tmem_wait_st();  // an aborted softmax warp may hold a pending store
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
template <int D, int BK>
cudaError_t launch_attn_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int BH,
                          cudaStream_t stream) {
    using Cfg = AttnCfg<D, BK>;
    static PerDeviceOnce configured;
    const int dev = PerDeviceOnce::current();
    if (!configured.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(vc_attn_kernel<D, BK, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(vc_attn_kernel<D, BK, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured.mark(dev);
    }
    dim3 grid((a.N + Cfg::BM - 1) / Cfg::BM, BH);
    if (a.tile_mask)
        vc_attn_kernel<D, BK, true><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tk, tv, a);
    else
        vc_attn_kernel<D, BK, false><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tk, tv, a);
    return cudaGetLastError();
}

cudaError_t launch_attn(int D, int BK, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int BH,
                        cudaStream_t stream) {
    if (D == 128 && BK == 128) return launch_attn_t<128, 128>(tk, tv, a, BH, stream);
    if (D == 128 && BK == 64) return launch_attn_t<128, 64>(tk, tv, a, BH, stream);
    if (D == 64 && BK == 128) return launch_attn_t<64, 128>(tk, tv, a, BH, stream);
    if (D == 64 && BK == 64) return launch_attn_t<64, 64>(tk, tv, a, BH, stream);
    return cudaErrorInvalidValue;
}

// ExpCast byte map, element-wise (the same packed device function the kernel
// uses; the second lane of the pair repeats the first).
__global__ void vc_expcast_kernel(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float cbm = cb[i] + kMagic;
        out[i] = (uint8_t)(expcast4(A[i], s[i], s[i], s[i], s[i], cbm) & 0xFFu);
    }
}

cudaError_t launch_expcast(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n,
                           cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const int64_t cap = 16LL * sm_count();
    const unsigned grid = (unsigned)((n + 255) / 256 < cap ? (n + 255) / 256 : cap);
    vc_expcast_kernel<<<grid, 256, 0, stream>>>(A, s, cb, out, n);
    return cudaGetLastError();
}

}  // namespace vc
