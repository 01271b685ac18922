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
// One CTA computes a 128-row query tile of one (b, h) against all T key tiles:
//   warp 0       TMA producer: Q tile once; K tile, V^T tile and block mean per
//                key tile through a STAGES-deep ring.
//   warp 1       TMEM owner and MMA issuer (one thread):
//                  S[t%2]  = Q K_t^T                       (kind::f8f6f4, TMEM fp32)
//                  O      += P_t V_t                       (accumulates over t)
//                  L[t%2]  = P_t 1   (row sums of the bytes' values, N = 16)
//   warps 2..5   softmax, one thread per query row: row max of S, integer row
//                reference M (raised online; a rise by k rescales O by 2^-k,
//                exactly), ExpCast bytes into shared memory as the A operand of
//                the PV MMA.
//   warps 6..9   correction, one thread per row: acc += l_t * mu_t (the block-
//                mean restore) and l += l_t, both rescaled with O; epilogue
//                O = (v_scale * O + acc) / l in bf16, original token order.
// Every wait is bounded (DevCtl); on a timeout the CTA drains its copies and
// MMAs, frees TMEM and exits with the status word set.
#include "vc_launch.cuh"

namespace vc {


template <int D, int BK>
struct AttnCfg {
    static constexpr int BM = 128;
    static constexpr int STAGES = 3;
    static constexpr int THREADS = 320;
    static constexpr int Q_BYTES = BM * D;
    static constexpr int K_BYTES = BK * D;
    static constexpr int V_BYTES = D * BK;
    static constexpr int P_BYTES = BM * BK;
    static constexpr int ONES_BYTES = 16 * BK;
    static constexpr int MU_BYTES = D * 4;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
    static constexpr int OFF_P = OFF_V + STAGES * V_BYTES;
    static constexpr int OFF_ONES = OFF_P + 2 * P_BYTES;
    static constexpr int OFF_MU = OFF_ONES + ONES_BYTES;
    static constexpr int OFF_KINC = OFF_MU + STAGES * MU_BYTES;
    static constexpr int OFF_BAR = OFF_KINC + 4 * BM * 4;
    // barrier slots
    static constexpr int B_QFULL = 0;
    static constexpr int B_KFULL = 1;
    static constexpr int B_KEMPTY = B_KFULL + STAGES;
    static constexpr int B_VFULL = B_KEMPTY + STAGES;
    static constexpr int B_VEMPTY = B_VFULL + STAGES;
    static constexpr int B_SFULL = B_VEMPTY + STAGES;
    static constexpr int B_SFREE = B_SFULL + 2;
    static constexpr int B_PFULL = B_SFREE + 2;
    static constexpr int B_PVDONE = B_PFULL + 2;
    static constexpr int B_LFREE = B_PVDONE + 2;
    static constexpr int B_KINC = B_LFREE + 2;
    static constexpr int B_MMADONE = B_KINC + 4;
    static constexpr int NBAR = B_MMADONE + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
    // TMEM columns
    static constexpr int O_COL = 0;
    static constexpr int S_COL0 = D;
    static constexpr int L_COL0 = D + 2 * BK;
    static constexpr int TMEM_USED = D + 2 * BK + 32;
    static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert((Q_BYTES % 1024) == 0 && (K_BYTES % 1024) == 0 && (P_BYTES % 1024) == 0 &&
                      (ONES_BYTES % 1024) == 0,
                  "swizzled tiles stay 1024-byte aligned");
};

__device__ __forceinline__ float exp2_neg_int(int k) {
    // 2^-k for an integer k >= 0, exactly (0 below the normal range).
    return k < 127 ? __uint_as_float((uint32_t)(127 - k) << 23) : 0.0f;
}

// Wait with a warp-uniform verdict: the warp continues only if every lane saw
// the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevCtl& ctl, volatile int* abort_flag) {
    const bool ok = mbar_wait(bar, parity, ctl, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies and
// MMAs before the CTA exits).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, const DevCtl& ctl) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if ((int64_t)(globaltimer() - t0) > ctl.limit_ns) {
            record_error(ctl, VC_ERR_DEVICE_TIMEOUT);
            return;
        }
    }
}

template <int D, int BK>
__global__ void __launch_bounds__(320, 1)
    vc_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs args) {
    using Cfg = AttnCfg<D, BK>;
    constexpr int STAGES = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * Cfg::BM;
    const int bh = blockIdx.y;
    const int N = args.N;
    const int T = args.T;

    auto bar = [&](int i) -> uint32_t { return base + Cfg::OFF_BAR + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
    int* kinc_ring = reinterpret_cast<int*>(smem + Cfg::OFF_KINC);

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        mbar_init(bar(Cfg::B_QFULL), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(Cfg::B_KFULL + s), 1);
            mbar_init(bar(Cfg::B_KEMPTY + s), 1);
            mbar_init(bar(Cfg::B_VFULL + s), 1);
            mbar_init(bar(Cfg::B_VEMPTY + s), 1 + 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(Cfg::B_SFULL + i), 1);
            mbar_init(bar(Cfg::B_SFREE + i), 4);
            mbar_init(bar(Cfg::B_PFULL + i), 4);
            mbar_init(bar(Cfg::B_PVDONE + i), 1);
            mbar_init(bar(Cfg::B_LFREE + i), 4);
        }
        for (int i = 0; i < 4; ++i) mbar_init(bar(Cfg::B_KINC + i), 4);
        mbar_init(bar(Cfg::B_MMADONE), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    {  // the constant "ones" B operand of the row-sum MMA: every byte is E4M3 1.0
        uint4* ones = reinterpret_cast<uint4*>(smem + Cfg::OFF_ONES);
        const uint4 v = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
        for (int i = threadIdx.x; i < Cfg::ONES_BYTES / 16; i += Cfg::THREADS) ones[i] = v;
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const DevCtl ctl = args.ctl;

    if (warp == 0) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            mbar_expect_tx_arrive(bar(Cfg::B_QFULL), Cfg::Q_BYTES);
            tma_load_3d(base + Cfg::OFF_Q, &tm_q, bar(Cfg::B_QFULL), 0, q0, bh);
            int issued_k = 0, issued_v = 0;
            for (int t = 0; t < T; ++t) {
                const int st = t % STAGES;
                const int n = t / STAGES;
                if (n > 0 && !mbar_wait(bar(Cfg::B_KEMPTY + st), (n - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(bar(Cfg::B_KFULL + st), Cfg::K_BYTES);
                tma_load_3d(base + Cfg::OFF_K + st * Cfg::K_BYTES, &tm_k, bar(Cfg::B_KFULL + st), 0, t * BK, bh);
                issued_k = t + 1;
                if (n > 0 && !mbar_wait(bar(Cfg::B_VEMPTY + st), (n - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(bar(Cfg::B_VFULL + st), Cfg::V_BYTES + Cfg::MU_BYTES);
                tma_load_3d(base + Cfg::OFF_V + st * Cfg::V_BYTES, &tm_v, bar(Cfg::B_VFULL + st), t * BK, 0, bh);
                bulk_load(base + Cfg::OFF_MU + st * Cfg::MU_BYTES, args.v_mean + ((size_t)bh * T + t) * D,
                          Cfg::MU_BYTES, bar(Cfg::B_VFULL + st));
                issued_v = t + 1;
            }
            // Drain: every copy issued has landed before the CTA may exit.  Only
            // the last STAGES tiles of each ring can still be in flight.
            drain_wait(bar(Cfg::B_QFULL), 0, ctl);
            for (int t = issued_k - STAGES < 0 ? 0 : issued_k - STAGES; t < issued_k; ++t)
                drain_wait(bar(Cfg::B_KFULL + t % STAGES), (t / STAGES) & 1, ctl);
            for (int t = issued_v - STAGES < 0 ? 0 : issued_v - STAGES; t < issued_v; ++t)
                drain_wait(bar(Cfg::B_VFULL + t % STAGES), (t / STAGES) & 1, ctl);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_e4m3_f32(BK);
            const uint32_t id_pv = idesc_e4m3_f32(D);
            const uint32_t id_l = idesc_e4m3_f32(16);
            const uint64_t dq = smem_desc(base + Cfg::OFF_Q, D);
            const uint64_t dones = smem_desc(base + Cfg::OFF_ONES, BK);
            bool ok = mbar_wait(bar(Cfg::B_QFULL), 0, ctl, abort_flag);
            auto issue_qk = [&](int t) -> bool {
                const int st = t % STAGES, sb = t & 1;
                if (!mbar_wait(bar(Cfg::B_KFULL + st), (t / STAGES) & 1, ctl, abort_flag)) return false;
                if (t >= 2 && !mbar_wait(bar(Cfg::B_SFREE + sb), ((t - 2) >> 1) & 1, ctl, abort_flag)) return false;
                tc_fence_after();
                const uint64_t dk = smem_desc(base + Cfg::OFF_K + st * Cfg::K_BYTES, D);
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    mma_f8(tmem + Cfg::S_COL0 + sb * BK, dq + 2 * kk, dk + 2 * kk, id_qk, kk > 0);
                mma_commit(bar(Cfg::B_SFULL + sb));
                mma_commit(bar(Cfg::B_KEMPTY + st));
                return true;
            };
            auto issue_pv = [&](int t) -> bool {
                const int st = t % STAGES, pb = t & 1;
                if (!mbar_wait(bar(Cfg::B_PFULL + pb), (t >> 1) & 1, ctl, abort_flag)) return false;
                if (!mbar_wait(bar(Cfg::B_VFULL + st), (t / STAGES) & 1, ctl, abort_flag)) return false;
                if (t >= 2 && !mbar_wait(bar(Cfg::B_LFREE + pb), ((t - 2) >> 1) & 1, ctl, abort_flag)) return false;
                tc_fence_after();
                const uint64_t dp = smem_desc(base + Cfg::OFF_P + pb * Cfg::P_BYTES, BK);
                const uint64_t dv = smem_desc(base + Cfg::OFF_V + st * Cfg::V_BYTES, BK);
#pragma unroll
                for (int kk = 0; kk < BK / 32; ++kk)
                    mma_f8(tmem + Cfg::O_COL, dp + 2 * kk, dv + 2 * kk, id_pv, (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < BK / 32; ++kk)
                    mma_f8(tmem + Cfg::L_COL0 + 16 * pb, dp + 2 * kk, dones + 2 * kk, id_l, kk > 0);
                mma_commit(bar(Cfg::B_PVDONE + pb));
                mma_commit(bar(Cfg::B_VEMPTY + st));
                return true;
            };
            if (ok) ok = issue_qk(0);
            for (int t = 0; ok && t < T; ++t) {
                if (t + 1 < T && !issue_qk(t + 1)) break;
                if (!issue_pv(t)) break;
            }
            mma_commit(bar(Cfg::B_MMADONE));
            drain_wait(bar(Cfg::B_MMADONE), 0, ctl);
        }
    } else if (warp < 6) {
        // -------------------------------------------------------- softmax
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_tmem = tmem + ((uint32_t)(qd * 32) << 16);
        const int qrow = q0 + row;
        const float sqv = qrow < N ? args.sq[(size_t)bh * N + qrow] : 0.0f;
        const float aq = __fmul_rn(args.kappa, sqv);
        const float c0 = 56.0f + (float)args.beta;
        uint8_t* pbuf = smem + Cfg::OFF_P;
        float M = 0.0f;
        float sk_next = args.k_scale[(size_t)bh * T];
        for (int t = 0; t < T; ++t) {
            const int sb = t & 1;
            const float sk = sk_next;
            if (t + 1 < T) sk_next = args.k_scale[(size_t)bh * T + t + 1];
            if (!warp_wait(bar(Cfg::B_SFULL + sb), (t >> 1) & 1, ctl, abort_flag)) break;
            tc_fence_after();
            float s[BK];
#pragma unroll
            for (int c = 0; c < BK / 32; ++c) tmem_ld32(lane_tmem + Cfg::S_COL0 + sb * BK + 32 * c, s + 32 * c);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_SFREE + sb));

            const int valid = N - t * BK;
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
            const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
            const float A = __fmul_rn(aq, sk);
            const float Mc = ceilf(__fmul_rn(__fmul_rn(A, mx), 0.125f));
            const float Mnew = t == 0 ? Mc : fmaxf(M, Mc);
            const int kinc = t == 0 ? 0 : (int)(Mnew - M);
            M = Mnew;
            const float cbm = (c0 - 8.0f * M) + kMagic;
            // P buffer sb was last read by the PV MMA of tile t-2.
            if (t >= 2 && !warp_wait(bar(Cfg::B_PVDONE + sb), ((t - 2) >> 1) & 1, ctl, abort_flag)) break;
            uint8_t* prow = pbuf + sb * Cfg::P_BYTES;
#pragma unroll
            for (int ch = 0; ch < BK / 16; ++ch) {
                uint32_t w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = ch * 16 + q * 4;
                    const float2 t01 = expcast_t2(A, s[j], s[j + 1], cbm);
                    const float2 t23 = expcast_t2(A, s[j + 2], s[j + 3], cbm);
                    w[q] = pack4_low_bytes(t01.x, t01.y, t23.x, t23.y);
                }
                *reinterpret_cast<uint4*>(prow + swz_offset(row, ch, BK)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (t > 0 && __any_sync(0xffffffffu, kinc > 0)) {
                // O holds PV of tiles < t: wait for it, then scale by 2^-kinc
                // (before this tile's PV, which waits on p_full below).
                if (!warp_wait(bar(Cfg::B_PVDONE + ((t - 1) & 1)), ((t - 1) >> 1) & 1, ctl, abort_flag)) break;
                tc_fence_after();
                const float f = exp2_neg_int(kinc);
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float o[32];
                    tmem_ld32(lane_tmem + Cfg::O_COL + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= f;
                    tmem_st32(lane_tmem + Cfg::O_COL + 32 * c, o);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            kinc_ring[(t & 3) * Cfg::BM + row] = kinc;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(Cfg::B_PFULL + sb));
                mbar_arrive(bar(Cfg::B_KINC + (t & 3)));
            }
        }
    } else {
        // -------------------------------------------------------- correction + epilogue
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_tmem = tmem + ((uint32_t)(qd * 32) << 16);
        const int qrow = q0 + row;
        float acc[D];
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = 0.0f;
        float l = 0.0f;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int st = t % STAGES;
            if (!(ok = warp_wait(bar(Cfg::B_KINC + (t & 3)), (t >> 2) & 1, ctl, abort_flag))) break;
            const int kinc = kinc_ring[(t & 3) * Cfg::BM + row];
            if (!(ok = warp_wait(bar(Cfg::B_PVDONE + (t & 1)), (t >> 1) & 1, ctl, abort_flag))) break;
            tc_fence_after();
            const float lb = tmem_ld1(lane_tmem + Cfg::L_COL0 + 16 * (t & 1));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_LFREE + (t & 1)));
            if (!(ok = warp_wait(bar(Cfg::B_VFULL + st), (t / STAGES) & 1, ctl, abort_flag))) break;
            if (kinc > 0) {
                const float f = exp2_neg_int(kinc);
#pragma unroll
                for (int c = 0; c < D; ++c) acc[c] *= f;
                l *= f;
            }
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
            l += lb;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_VEMPTY + st));
        }
        if (ok && T > 0) {
            // The last PV (tile T-1) has completed, so O is final.
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const float* vsc = args.v_scale + (size_t)bh * D;
            __nv_bfloat16* orow = args.out + ((size_t)bh * N + qrow) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tmem_ld32(lane_tmem + Cfg::O_COL + 32 * c, o);
                tmem_wait_ld();
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c0i = 32 * c + 2 * i;
                    const float x0 = (vsc[c0i] * o[2 * i] + acc[c0i]) * inv_l;
                    const float x1 = (vsc[c0i + 1] * o[2 * i + 1] + acc[c0i + 1]) * inv_l;
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                    packed[i] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                if (qrow < N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                }
            }
        }
    }

    // ------------------------------------------------------------ teardown
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
cudaError_t launch_attn_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                          int BH, cudaStream_t stream) {
    using Cfg = AttnCfg<D, BK>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(vc_attn_kernel<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    dim3 grid((a.N + Cfg::BM - 1) / Cfg::BM, BH);
    vc_attn_kernel<D, BK><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

cudaError_t launch_attn(int D, int BK, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const AttnArgs& a, int BH, cudaStream_t stream) {
    if (D == 128 && BK == 128) return launch_attn_t<128, 128>(tq, tk, tv, a, BH, stream);
    if (D == 128 && BK == 64) return launch_attn_t<128, 64>(tq, tk, tv, a, BH, stream);
    if (D == 64 && BK == 128) return launch_attn_t<64, 128>(tq, tk, tv, a, BH, stream);
    if (D == 64 && BK == 64) return launch_attn_t<64, 64>(tq, tk, tv, a, BH, stream);
    return cudaErrorInvalidValue;
}

// ExpCast byte map, element-wise (the same packed device function the kernel
// uses; the second lane of the pair repeats the first).
__global__ void vc_expcast_kernel(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float cbm = cb[i] + kMagic;
        const float2 t = expcast_t2(A[i], s[i], s[i], cbm);
        out[i] = (uint8_t)(__float_as_uint(t.x) & 0xFFu);
    }
}

cudaError_t launch_expcast(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n,
                           cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
    vc_expcast_kernel<<<grid, 256, 0, stream>>>(A, s, cb, out, n);
    return cudaGetLastError();
}

}  // namespace vc
