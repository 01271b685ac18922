// vc_attn4.cu -- the 4-bit path of the attention forward: ExpCast on FP8
// scores as in vc_attn.cu, then a PV product of NVFP4 operands on sm_100a
// tensor cores (tcgen05 kind::mxf4nvf4, block16 UE4M3 scales).
//
// Method: the zerohour.day summary gives NVFP4 beside E4M3 as a format of
// the per-channel V residual.  A kind::mxf4nvf4 product needs
// both operands in E2M1, so P is re-coded to NVFP4 in the softmax stage: each
// run of 16 keys of a row takes the UE4M3 scale E4M3(max/6) of its ExpCast
// values, and each value the E2M1 code of p * (1/scale).  QK^T stays FP8.
//
// One CTA computes a 128-row query tile of one (b, h) against all T key tiles
// of 128 keys.
//   TMEM (columns): S0, S1 [128 each] | O [D + 16] | Q [D/4] |
//                   SFA [2 buffers x 2 MMAs x 4] | SFB [2 buffers x 2 MMAs x NBP]
//                   O's column D accumulates the running row sum l: the V^T
//                   tile is followed by 16 rows of E2M1 ones with scale 1.
//   SMEM: K ring (E4M3), V^T ring (E2M1, 64-byte rows), the V block scales and
//         block means per stage, and two P tiles (E2M1, 64-byte rows, written
//         by the softmax warps in the layout TMA would give: 64-byte swizzle).
//   warp 0      TMA producer: K tile, V^T tile, V block scales and block mean
//               per key tile through a STAGES-deep ring.
//   warp 1      TMEM owner and MMA issuer (one elected lane):
//                 S[t%2] = Q K_t^T                 (kind::f8f6f4, A = Q in TMEM)
//                 [O|l] += P_t [V_t|1]             (kind::mxf4nvf4, A and B in SMEM,
//                                                   two MMAs of K = 64)
//   warps 2..5  softmax, one warp per TMEM lane quadrant, a thread per query
//               row: row max, integer row reference M, ExpCast codes, NVFP4
//               re-coding of P into SMEM; P's block scales go through shared
//               memory so that every warp can write all four lane-quadrant
//               copies the tensor core reads.  On a rise of M: O scaled by 2^-k.
//   warps 6..9  correction, one warp per quadrant: l_t from O's column D, the
//               V block scales of the next tile into TMEM (four copies) before
//               that tile's PV, acc += l_t * mu_t; epilogue as in vc_attn.cu.
// Every wait is bounded (DevCtl); on a timeout the CTA drains its copies and
// MMAs, frees TMEM and exits with the status word set.
#include "vc_launch.cuh"

namespace vc {

template <int D>
struct Attn4Cfg {
    static constexpr int BM = 128;
    static constexpr int BK = 128;
    static constexpr int G = BK / 16;           // NVFP4 blocks per row of a tile
    static constexpr int STAGES = 4;
    static constexpr int THREADS = 320;         // 10 warps
    static constexpr int K_BYTES = BK * D;      // E4M3 K tile
    static constexpr int VROW = BK / 2;         // bytes of a V^T row (E2M1)
    static constexpr int V_BYTES = D * VROW;    // the TMA-loaded V^T tile
    static constexpr int VX_BYTES = (D + 16) * VROW;  // + 16 rows of ones (the l column)
    static constexpr int SFB_BYTES = D * G;     // V block scales of a tile
    static constexpr int MU_BYTES = D * 4;
    static constexpr int P_BYTES = BM * VROW;   // an E2M1 P tile
    static constexpr int NB = (D + 16 + 31) / 32;  // SFB columns per MMA
    static constexpr int NBP = (NB + 3) / 4 * 4;    // ... each MMA's block starting on a 4-column boundary
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
    static constexpr int OFF_P = OFF_V + STAGES * VX_BYTES;
    static constexpr int OFF_SFB = OFF_P + 2 * P_BYTES;
    static constexpr int OFF_MU = OFF_SFB + STAGES * SFB_BYTES;
    static constexpr int OFF_SFA = OFF_MU + STAGES * MU_BYTES;  // [parity][2][BM] words
    static constexpr int OFF_KINC = OFF_SFA + 2 * 2 * BM * 4;
    static constexpr int OFF_PLUT = OFF_KINC + 4 * BM * 4;  // 128 P block-scale entries
    static constexpr int OFF_BAR = OFF_PLUT + 128 * 8;
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
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    // TMEM columns
    static constexpr int S_COL0 = 0;
    static constexpr int O_COL = 2 * BK;
    static constexpr int L_COL = O_COL + D;
    static constexpr int Q_COL = O_COL + D + 16;
    static constexpr int SFA_COL = Q_COL + D / 4;
    static constexpr int SFB_COL = SFA_COL + 2 * 2 * 4;
    static constexpr int TMEM_USED = SFB_COL + 2 * 2 * NBP;
    static constexpr int TMEM_COLS = 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert(SFA_COL % 4 == 0 && SFB_COL % 4 == 0, "scale-factor blocks on 4-column boundaries");
    static_assert((K_BYTES % 1024) == 0 && (VX_BYTES % 1024) == 0 && (P_BYTES % 1024) == 0,
                  "swizzled tiles stay 1024-byte aligned");
};

// Barrier of the four softmax warps (named barrier 1, 128 threads) that also
// ANDs a verdict across them: all four see the same result, so a warp never
// waits there for one that has left.
__device__ __forceinline__ bool softmax_sync_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// The NVFP4 block scale of P depends only on the block's largest ExpCast code
// m (E4M3 codes increase with their values): its UE4M3 code E4M3(value(m)/6)
// and the reciprocal of its value, rounded to fp32, times 2^60 (0 for a zero
// scale).  One entry per code, built once per CTA with the same divide and
// reciprocal the block coder would use.
struct PScaleEntry {
    uint32_t sc;
    float r60;
};

__device__ __forceinline__ PScaleEntry p_scale_entry(uint32_t m) {
    const uint32_t sc = (uint32_t)(e4m3x2(__fdiv_rn(e4m3_to_f32(m), 6.0f), 0.0f) & 0xFF);
    const float sv = e4m3_to_f32(sc);
    return PScaleEntry{sc, sv > 0.0f ? __fmul_rn(__frcp_rn(sv), 0x1p60f) : 0.0f};
}

// One 16-key NVFP4 block of P from the ExpCast codes, given as the floats
// w[e] = code * 2^-149 (whose bit patterns are the codes, ordered as the
// codes): the UE4M3 scale E4M3(max/6) and the E2M1 codes of p * (1/scale),
// p the E4M3 value, the product rounded once in fp32 as (p 2^-60)(r 2^60),
// both factors exact.  A zero scale codes zeros.
__device__ __forceinline__ void p_block_nvfp4(const float* w, const PScaleEntry* lut, uint32_t& w0, uint32_t& w1,
                                              uint32_t& scale) {
    const float m5[5] = {fmax3(w[0], w[1], w[2]), fmax3(w[3], w[4], w[5]), fmax3(w[6], w[7], w[8]),
                         fmax3(w[9], w[10], w[11]), fmax3(w[12], w[13], w[14])};
    const float mx = fmaxf(fmax3(m5[0], m5[1], m5[2]), fmax3(m5[3], m5[4], w[15]));
    const PScaleEntry ent = lut[__float_as_uint(mx) & 127u];
    const float2 k60 = make_float2(0x1p60f, 0x1p60f), r = make_float2(ent.r60, ent.r60);
    float x[16];
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
        const float2 p = make_float2(__uint_as_float(__float_as_uint(w[e]) << 20),
                                     __uint_as_float(__float_as_uint(w[e + 1]) << 20));
        const float2 y = fmul2(fmul2(p, k60), r);
        x[e] = y.x;
        x[e + 1] = y.y;
    }
    w0 = e2m1x8(x);
    w1 = e2m1x8(x + 8);
    scale = ent.sc;
}

// ExpCast codes of two scores, clamped at 0: t = A*s + cbm rounds A*s + cb to
// the integer n once (cbm = cb + 1.5*2^23), and sat(t*2^-149 - 1.5*2^-126) is
// max(n, 0)*2^-149 exactly, whose bit pattern is max(n, 0).
__device__ __forceinline__ void expcast_codes2(float A, float s0, float s1, float cbm, float& w0, float& w1) {
    const float2 t = ffma2(make_float2(A, A), make_float2(s0, s1), make_float2(cbm, cbm));
    asm("fma.rn.sat.f32 %0, %1, 0f00000001, 0f80C00000;" : "=f"(w0) : "f"(t.x));
    asm("fma.rn.sat.f32 %0, %1, 0f00000001, 0f80C00000;" : "=f"(w1) : "f"(t.y));
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    vc_attn4_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const AttnArgs args) {
    using Cfg = Attn4Cfg<D>;
    constexpr int STAGES = Cfg::STAGES;
    constexpr int BK = Cfg::BK;
    constexpr int G = Cfg::G;
    constexpr int NB = Cfg::NB;
    constexpr int NBP = Cfg::NBP;
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
    const int T = args.T;

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
            // P(t) and its scales posted by the 4 softmax warps; l(t-1) read
            // and SFB(t) written by the 4 correction warps
            mbar_init(bar(Cfg::B_PFULL + i), 4 + 4);
            mbar_init(bar(Cfg::B_PVDONE + i), 1);
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
    {  // rows D..D+15 of every V stage: E2M1 1.0 (code 2), so the PV MMA also sums P
        constexpr int PER = 16 * Cfg::VROW / 16;  // uint4 per stage
        const uint4 v = make_uint4(0x22222222u, 0x22222222u, 0x22222222u, 0x22222222u);
        for (int i = threadIdx.x; i < STAGES * PER; i += Cfg::THREADS)
            reinterpret_cast<uint4*>(smem + Cfg::OFF_V + (i / PER) * Cfg::VX_BYTES + Cfg::V_BYTES)[i % PER] = v;
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
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int issued_k = 0, issued_v = 0;
            for (int t = 0; t < T; ++t) {
                const int st = t % STAGES;
                const int n = t / STAGES;
                if (n > 0 && !mbar_wait(bar(Cfg::B_KEMPTY + st), (n - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(bar(Cfg::B_KFULL + st), Cfg::K_BYTES);
                tma_load_3d(base + Cfg::OFF_K + st * Cfg::K_BYTES, &tm_k, bar(Cfg::B_KFULL + st), 0, t * BK, bh);
                issued_k = t + 1;
                if (n > 0 && !mbar_wait(bar(Cfg::B_VEMPTY + st), (n - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(bar(Cfg::B_VFULL + st), Cfg::V_BYTES + Cfg::SFB_BYTES + Cfg::MU_BYTES);
                tma_load_3d(base + Cfg::OFF_V + st * Cfg::VX_BYTES, &tm_v, bar(Cfg::B_VFULL + st), t * Cfg::VROW, 0,
                            bh);
                bulk_load(base + Cfg::OFF_SFB + st * Cfg::SFB_BYTES, args.v_bscale + ((size_t)bh * T + t) * Cfg::SFB_BYTES,
                          Cfg::SFB_BYTES, bar(Cfg::B_VFULL + st));
                bulk_load(base + Cfg::OFF_MU + st * Cfg::MU_BYTES, args.v_mean + ((size_t)bh * T + t) * D,
                          Cfg::MU_BYTES, bar(Cfg::B_VFULL + st));
                issued_v = t + 1;
            }
            for (int t = issued_k - STAGES < 0 ? 0 : issued_k - STAGES; t < issued_k; ++t)
                drain_wait(bar(Cfg::B_KFULL + t % STAGES), (t / STAGES) & 1, ctl);
            for (int t = issued_v - STAGES < 0 ? 0 : issued_v - STAGES; t < issued_v; ++t)
                drain_wait(bar(Cfg::B_VFULL + t % STAGES), (t / STAGES) & 1, ctl);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        const uint32_t id_qk = idesc_e4m3_f32(BK);
        const uint32_t id_pv = idesc_nvf4_f32(D + 16);
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
            // p_full(t): P(t) and SFA(t) from the softmax warps, l(t-1) read and
            // SFB(t) written by the correction warps, which waited for V(t) to
            // land before writing SFB(t): one wait here
            if (!warp_wait(bar(Cfg::B_PFULL + pb), (t >> 1) & 1, ctl, abort_flag)) return false;
            tc_fence_after();
            const uint64_t dp = smem_desc(base + Cfg::OFF_P + pb * Cfg::P_BYTES, Cfg::VROW);
            const uint64_t dv = smem_desc(base + Cfg::OFF_V + st * Cfg::VX_BYTES, Cfg::VROW);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)  // K = 64 keys an MMA: 32 bytes of each row
                mma_nvf4_ss_warp(tmem + Cfg::O_COL, dp + 2 * kk, dv + 2 * kk, id_pv,
                                 tmem + Cfg::SFA_COL + pb * 8 + kk * 4, tmem + Cfg::SFB_COL + pb * 2 * NBP + kk * NBP,
                                 (t > 0 || kk > 0) ? 1u : 0u);
            mma_commit_warp(bar(Cfg::B_PVDONE + pb));
            mma_commit_warp(bar(Cfg::B_VEMPTY + st));
            return true;
        };
        if (ok) ok = issue_qk(0);
        for (int t = 0; ok && t < T; ++t) {
            if (t + 1 < T && !issue_qk(t + 1)) break;
            if (!issue_pv(t)) break;
        }
        mma_commit_warp(bar(Cfg::B_MMADONE));
        drain_wait(bar(Cfg::B_MMADONE), 0, ctl);
    } else if (warp < 6) {
        // -------------------------------------------------------- softmax
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
        uint32_t* sfa_x = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_SFA);  // [parity][MMA][row]
        PScaleEntry* plut = reinterpret_cast<PScaleEntry*>(smem + Cfg::OFF_PLUT);
        plut[row] = p_scale_entry((uint32_t)row);  // the 128 softmax threads, one code each
        bool run = softmax_sync_and(true);
        float M = 0.0f;
        float sk_next = args.k_scale[(size_t)bh * T];
        for (int t = 0; run && t < T; ++t) {
            const int sb = t & 1;
            const float sk = sk_next;
            if (t + 1 < T) sk_next = args.k_scale[(size_t)bh * T + t + 1];
            const bool ok = warp_wait(bar(Cfg::B_SFULL + sb), (t >> 1) & 1, ctl, abort_flag);
            int kinc = 0;
            if (ok) {
                tc_fence_after();
                float s[BK];
#pragma unroll
                for (int c = 0; c < BK / 32; ++c) tmem_ld32(lane_tmem + Cfg::S_COL0 + sb * BK + 32 * c, s + 32 * c);
                tmem_wait_ld();
                const int valid = N - t * BK;
                if (valid < BK) {
#pragma unroll
                    for (int j = 0; j < BK; ++j)
                        if (j >= valid) s[j] = -INFINITY;
                }
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
                kinc = t == 0 ? 0 : (int)(Mnew - M);
                M = Mnew;
                const float cbm = (c0 - 8.0f * M) + kMagic;
                kinc_ring[(t & 3) * Cfg::BM + row] = kinc;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(Cfg::B_KINC + (t & 3)));
                // P slot sb (SMEM tile and SFA columns) was last read by PV(t-2),
                // complete: QK(t), whose commit s_full(t) this warp waited for,
                // was issued after it by the same thread.
                uint8_t* ptile = smem + Cfg::OFF_P + sb * Cfg::P_BYTES;
                uint32_t sfw[2] = {0u, 0u};
#pragma unroll
                for (int ch = 0; ch < Cfg::VROW / 16; ++ch) {  // 32 keys -> one 16-byte chunk of the row
                    uint32_t pw[4];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int g = 2 * ch + h;
                        float wc[16];
#pragma unroll
                        for (int e = 0; e < 16; e += 2)
                            expcast_codes2(A, s[16 * g + e], s[16 * g + e + 1], cbm, wc[e], wc[e + 1]);
                        uint32_t sc;
                        p_block_nvfp4(wc, plut, pw[2 * h], pw[2 * h + 1], sc);
                        sfw[g / 4] |= sc << (8 * (g % 4));
                    }
                    *reinterpret_cast<uint4*>(ptile + swz_offset(row, ch, Cfg::VROW)) =
                        make_uint4(pw[0], pw[1], pw[2], pw[3]);
                }
                sfa_x[(sb * 2 + 0) * Cfg::BM + row] = sfw[0];
                sfa_x[(sb * 2 + 1) * Cfg::BM + row] = sfw[1];
                fence_proxy_async_smem();  // the P tile is read by the tensor core
            }
            // Every row's P block scales are in shared memory (and every warp
            // passed its wait), or all four warps stop here together.
            if (!softmax_sync_and(ok)) break;
            {   // SFA(t): the scales of rows l, 32+l, 64+l, 96+l of both MMAs, in
                // this warp's lane quadrant (the tensor core reads every quadrant)
                uint32_t sw[8];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sw[kk * 4 + c] = sfa_x[(sb * 2 + kk) * Cfg::BM + 32 * c + lane];
                tmem_st8(lane_tmem + Cfg::SFA_COL + sb * 8, sw);
            }
            if (t > 0 && __any_sync(0xffffffffu, kinc > 0)) {
                // O holds PV of tiles < t: wait for it, then scale O by 2^-kinc
                // (l is scaled by the correction warps).  A failed wait skips the
                // work; the warps stop together at the next tile's barrier.
                if (warp_wait(bar(Cfg::B_PVDONE + ((t - 1) & 1)), ((t - 1) >> 1) & 1, ctl, abort_flag)) {
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
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_PFULL + sb));
        }
    } else {
        // -------------------------------------------------------- correction + epilogue
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_tmem = tmem + ((uint32_t)(qd * 32) << 16);
        const int qrow = q0 + row;
        // SFB(t) into TMEM buffer t%2, this warp's lane quadrant: lane l holds
        // rows l + 32c of B (channels, then the 16 ones rows with scale 1.0)
        auto write_sfb = [&](int t) {
            const uint8_t* sfb = smem + Cfg::OFF_SFB + (t % STAGES) * Cfg::SFB_BYTES;  // [channel][G]
            const uint32_t col = lane_tmem + Cfg::SFB_COL + (t & 1) * 2 * NBP;
#pragma unroll
            for (int c = 0; c < NB; ++c) {
                const int n = 32 * c + lane;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint32_t w = n < D ? *reinterpret_cast<const uint32_t*>(sfb + n * G + 4 * kk)
                                             : (n < D + 16 ? 0x38383838u : 0u);
                    tmem_st1(col + kk * NBP + c, __uint_as_float(w));
                }
            }
        };
        float acc[D];
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = 0.0f;
        float l = 0.0f;
        bool ok = T == 0 || warp_wait(bar(Cfg::B_VFULL + 0), 0, ctl, abort_flag);
        if (ok && T > 0) {  // SFB(0) before PV(0), which waits on p_full(0)
            write_sfb(0);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Cfg::B_PFULL + 0));
        }
        ok = ok && (T == 0 || warp_wait(bar(Cfg::B_KINC + 0), 0, ctl, abort_flag));
        int kinc = 0;
        for (int t = 0; ok && t < T; ++t) {
            const int st = t % STAGES;
            if (!(ok = warp_wait(bar(Cfg::B_PVDONE + (t & 1)), (t >> 1) & 1, ctl, abort_flag))) break;
            tc_fence_after();
            const float lt = tmem_ld1(lane_tmem + Cfg::L_COL);
            tmem_wait_ld();
            const int kt = kinc;
            if (t + 1 < T) {
                // before PV(t+1), which waits for p_full(t+1): l(t) * 2^-k(t+1) into
                // O's l column, and the V block scales of tile t+1 (their TMEM
                // buffer was last read by PV(t-1), complete with PV(t))
                const int tn = t + 1;
                if (!(ok = warp_wait(bar(Cfg::B_KINC + (tn & 3)), (tn >> 2) & 1, ctl, abort_flag))) break;
                kinc = kinc_ring[(tn & 3) * Cfg::BM + row];
                if (__any_sync(0xffffffffu, kinc > 0)) tmem_st1(lane_tmem + Cfg::L_COL, lt * exp2_neg_int(kinc));
                if (!(ok = warp_wait(bar(Cfg::B_VFULL + tn % STAGES), (tn / STAGES) & 1, ctl, abort_flag))) break;
                write_sfb(tn);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && t + 1 < T) mbar_arrive(bar(Cfg::B_PFULL + ((t + 1) & 1)));
            if (!(ok = warp_wait(bar(Cfg::B_VFULL + st), (t / STAGES) & 1, ctl, abort_flag))) break;
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
        if (ok && T > 0) {
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
        }
    }

    // ------------------------------------------------------------ teardown
    if (warp >= 2) tmem_wait_st();  // an aborted warp may hold a pending TMEM store
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
template <int D>
cudaError_t launch_attn4_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int BH,
                           cudaStream_t stream) {
    using Cfg = Attn4Cfg<D>;
    static PerDeviceOnce configured;
    const int dev = PerDeviceOnce::current();
    if (!configured.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(vc_attn4_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured.mark(dev);
    }
    dim3 grid((a.N + Cfg::BM - 1) / Cfg::BM, BH);
    vc_attn4_kernel<D><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tk, tv, a);
    return cudaGetLastError();
}

cudaError_t launch_attn4(int D, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int BH,
                         cudaStream_t stream) {
    if (D == 128) return launch_attn4_t<128>(tk, tv, a, BH, stream);
    if (D == 64) return launch_attn4_t<64>(tk, tv, a, BH, stream);
    return cudaErrorInvalidValue;
}

}  // namespace vc
