// vc_prep.cu -- V-Smooth prep and Q quantisation on sm_100a.
//
// V-Smooth (chooseai.io news 7051, section "核心方法之一：V-Smooth 把 value 的
// 离群值收拢"; zerohour.day key facts): a lightweight k-means puts similar value
// tokens into the same hardware block; the block mean is subtracted and kept
// in high precision; the residual is quantised to E4M3 with per-channel scales.
// K moves with V so every (k_j, v_j) pair stays together.
//
// Kernels, per call, for all (b, h) at once:
//   km_init                   strided centroid init c_k = v[floor(k N / C)]
//   per pass: km_assign       labels = argmin_k |v - c_k|^2 (fp32, ties -> lowest k),
//                             per-(cluster, 128-token block) histogram, change count
//             km_scan         exclusive scan -> stable positions; a head whose labels
//                             did not change is final (its later passes would repeat)
//             km_scatter      perm[position] = token (stable within a cluster)
//             km_update       fp64 member sums over each cluster's contiguous range
//             km_finalize     c_k = sum / count (empty clusters keep c_k)
//   prep_kv_block             per block: K amax scale + E4M3 K, V block mean (fp64 sum),
//                             residual channel amax
//   prep_v_quant              per-channel residual scale, E4M3 residual, transposed
//   quant_q                   per-token E4M3 Q (used by the attention call)
#include <math.h>

#include "vc_launch.cuh"

namespace vc {


__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }
__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------------ k-means
// Centroids live as bf16 hi/lo pairs, row-major [BH, Cp, D] (Cp = C rounded up
// to 16; pad rows are zero), plus fp32 squared norms [BH, Cp]: v.c is computed
// on tensor cores as v.hi + v.lo (v is exact in bf16), so the distance
// |c|^2 - 2 v.c carries about 2^-16 relative error in c.
__device__ __forceinline__ void store_centroid(float c, __nv_bfloat16* hi, __nv_bfloat16* lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(c);
    *hi = h;
    *lo = __float2bfloat16_rn(c - __bfloat162float(h));
}

// Sum over the D threads of a block (D = blockDim.x, 64 or 128).
__device__ __forceinline__ float block_sum_d(float x, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    float t = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    return t;
}

__global__ void km_init(const __nv_bfloat16* __restrict__ V, __nv_bfloat16* __restrict__ c_hi,
                        __nv_bfloat16* __restrict__ c_lo, float* __restrict__ cnorm, double* __restrict__ cent64,
                        double* __restrict__ sums, KmState* __restrict__ state, uint32_t* __restrict__ vamax, int N,
                        int C, int Cp, int D) {
    __shared__ float red[4];
    const int k = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
    const size_t row = ((size_t)bh * Cp + k) * D + c;
    float x = 0.0f;
    if (k < C) {
        const int64_t src = ((int64_t)k * N) / C;
        x = bf2f(V[((size_t)bh * N + src) * D + c]);
        sums[((size_t)bh * C + k) * D + c] = 0.0;
        cent64[((size_t)bh * C + k) * D + c] = (double)x;
    }
    c_hi[row] = __float2bfloat16_rn(x);
    c_lo[row] = __float2bfloat16_rn(0.0f);
    const float nrm = block_sum_d(x * x, red);
    if (c == 0) cnorm[(size_t)bh * Cp + k] = nrm;
    if (k == 0) {
        vamax[(size_t)bh * D + c] = 0u;
        if (c == 0) state[bh] = KmState{0, 0, 0, 0};
    }
}

constexpr int KM_TOK = 128;  // tokens per assign block (the MMA's M)

// Assignment pass on tensor cores: one CTA = 128 tokens of one head.
//   S[token, k] = v . c_hi + v . c_lo   (kind::f16, bf16 x bf16 -> fp32 in TMEM)
//   label = argmin_k (|c_k|^2 - 2 S[token, k]), ties to the lowest k.
template <int D>
__global__ void __launch_bounds__(128) km_assign(const __grid_constant__ CUtensorMap tm_v,
                                                 const __grid_constant__ CUtensorMap tm_chi,
                                                 const __grid_constant__ CUtensorMap tm_clo,
                                                 const float* __restrict__ cnorm, const double* __restrict__ cent64,
                                                 const __nv_bfloat16* __restrict__ V, int32_t* __restrict__ labels,
                                                 int32_t* __restrict__ hist, KmState* __restrict__ state, int N, int C,
                                                 int Cp, int it, DevCtl ctl) {
    constexpr int A_BYTES = KM_TOK * D * 2;
    const int bh = blockIdx.y, blk = blockIdx.x, nblk = gridDim.x;
    // both uniform over the CTA, before any barrier or TMEM use
    if (ctl_failed(ctl.status) || state[bh].done) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const int B_BYTES = Cp * D * 2;
    const uint32_t sA = base, sBh = base + A_BYTES, sBl = sBh + B_BYTES;
    float* cn_s = reinterpret_cast<float*>(smem + A_BYTES + 2 * B_BYTES);
    int* hist_s = reinterpret_cast<int*>(cn_s + 256);
    uint64_t* bars = reinterpret_cast<uint64_t*>(hist_s + 256);  // [0] loads, [1] mma
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int n0 = blk * KM_TOK;
    const uint32_t ncols = Cp <= 32 ? 32 : (Cp <= 64 ? 64 : (Cp <= 128 ? 128 : 256));
    const uint32_t bar_ld = smem_u32(&bars[0]), bar_mma = smem_u32(&bars[1]);

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), ncols);
        tmem_relinquish();
    }
    for (int k = tid; k < Cp; k += 128) cn_s[k] = cnorm[(size_t)bh * Cp + k];
    for (int k = tid; k < C; k += 128) hist_s[k] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (tid == 0) {
        mbar_expect_tx_arrive(bar_ld, A_BYTES + 2 * B_BYTES);
#pragma unroll
        for (int kc = 0; kc < D / 64; ++kc) {
            tma_load_3d(sA + kc * (KM_TOK * 128), &tm_v, bar_ld, 64 * kc, n0, bh);
            tma_load_3d(sBh + kc * (Cp * 128), &tm_chi, bar_ld, 64 * kc, 0, bh);
            tma_load_3d(sBl + kc * (Cp * 128), &tm_clo, bar_ld, 64 * kc, 0, bh);
        }
        ok = mbar_wait(bar_ld, 0, ctl, abort_flag);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(Cp);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk & 3) * 32;
                const uint64_t da = smem_desc(sA + (kk >> 2) * (KM_TOK * 128) + off, 128);
                const uint64_t dh = smem_desc(sBh + (kk >> 2) * (Cp * 128) + off, 128);
                mma_bf16(tmem, da, dh, idesc, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk & 3) * 32;
                const uint64_t da = smem_desc(sA + (kk >> 2) * (KM_TOK * 128) + off, 128);
                const uint64_t dl = smem_desc(sBl + (kk >> 2) * (Cp * 128) + off, 128);
                mma_bf16(tmem, da, dl, idesc, 1u);
            }
        }
        mma_commit(bar_mma);  // also covers the case of no MMA issued
    }
    ok = __all_sync(0xffffffffu, mbar_wait(bar_mma, 0, ctl, abort_flag));
    int changed = 0;
    if (ok && !*abort_flag) {
        tc_fence_after();
        const uint32_t lane_tmem = tmem + ((uint32_t)(warp * 32) << 16);
        // pass 1: tensor-core distances |c|^2 - 2 v.c; best and runner-up
        float best = INFINITY, second = INFINITY;
        int bestk = 0;
        for (int k0 = 0; k0 < Cp; k0 += 16) {
            float dot[16];
            tmem_ld16(lane_tmem + k0, dot);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int k = k0 + j;
                const float dist = cn_s[k] - 2.0f * dot[j];
                if (k < C) {
                    if (dist < best) {
                        second = best;
                        best = dist;
                        bestk = k;
                    } else if (dist < second) {
                        second = dist;
                    }
                }
            }
        }
        // Error bound of the tensor-core distance: bf16 hi/lo centroids carry
        // 2^-18 relative error and the fp32 accumulation at most 2^-15 of
        // sum |v_c c_c|, so |err| <= 2^-14 (|v| + |c|)^2.  Candidates within
        // the margin are decided again in fp64, exactly as the Lloyd step
        // defines the distance (sum over channels, in order, of (v - c)^2).
        float vn2 = 0.0f;
        {
            const uint8_t* arow = smem + tid * 128;
#pragma unroll
            for (int kc = 0; kc < D / 64; ++kc)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(arow + kc * (KM_TOK * 128) + ((ch ^ (tid & 7)) << 4));
                    const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                    for (int e = 0; e < 8; ++e) vn2 = fmaf(bf2f(hv[e]), bf2f(hv[e]), vn2);
                }
        }
        float cmax2 = 0.0f;
        for (int k = 0; k < C; ++k) cmax2 = fmaxf(cmax2, cn_s[k]);
        const float rad = sqrtf(vn2) + sqrtf(cmax2);
        const float margin = ldexpf(rad * rad, -12);
        const bool valid_tok = n0 + tid < N;
        const bool refine = valid_tok && C > 1 && (second - best) <= margin;
        if (__any_sync(0xffffffffu, refine)) {
            // The warp evaluates each candidate of each refining lane together:
            // every lane sums (v - c)^2 over D/32 channels in fp64, then a
            // butterfly adds the lanes.  Candidates go in ascending k with a
            // strict comparison, so ties keep the lowest k.
            constexpr int CPL = D / 32;  // channels per lane
            const int lane = tid & 31;
            const float lim = best + margin;
            double dbest = INFINITY;
            int kbest = bestk;
            for (int k0 = 0; k0 < Cp; k0 += 16) {
                float dot[16];
                tmem_ld16(lane_tmem + k0, dot);
                tmem_wait_ld();
                uint32_t cm = 0;
                if (refine) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (k0 + j < C && cn_s[k0 + j] - 2.0f * dot[j] <= lim) cm |= 1u << j;
                }
                uint32_t lanes = __ballot_sync(0xffffffffu, cm != 0);
                while (lanes) {
                    const int src = __ffs(lanes) - 1;
                    lanes &= lanes - 1;
                    uint32_t m = __shfl_sync(0xffffffffu, cm, src);
                    const int r = warp * 32 + src;  // the source lane's token row in the tile
                    const int c0 = lane * CPL;
                    const uint8_t* vp = smem + (c0 / 64) * (KM_TOK * 128) + r * 128 +
                                        ((((c0 % 64) / 8) ^ (r & 7)) << 4) + (c0 % 8) * 2;
                    float vx[CPL];
                    if constexpr (CPL == 4) {
                        const uint2 raw = *reinterpret_cast<const uint2*>(vp);
                        const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                        for (int e = 0; e < 4; ++e) vx[e] = bf2f(hv[e]);
                    } else {
                        const uint32_t raw = *reinterpret_cast<const uint32_t*>(vp);
                        const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                        for (int e = 0; e < CPL; ++e) vx[e] = bf2f(hv[e]);
                    }
                    while (m) {
                        const int k = k0 + __ffs(m) - 1;
                        m &= m - 1;
                        const double* crow = cent64 + ((size_t)bh * C + k) * D + c0;
                        double part = 0.0;
#pragma unroll
                        for (int e = 0; e < CPL; ++e) {
                            const double diff = __dsub_rn((double)vx[e], crow[e]);
                            part = __dadd_rn(part, __dmul_rn(diff, diff));
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) part = __dadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
                        if (lane == src && part < dbest) {
                            dbest = part;
                            kbest = k;
                        }
                    }
                }
            }
            if (refine) bestk = kbest;
        }
        if (n0 + tid < N) {
            int32_t* lp = labels + (size_t)bh * N + n0 + tid;
            if (it == 0 || *lp != bestk) changed = 1;
            *lp = bestk;
            atomicAdd(&hist_s[bestk], 1);
        }
    }
    changed = __reduce_add_sync(0xffffffffu, changed);
    if ((tid & 31) == 0 && changed) atomicAdd(&state[bh].changed, changed);
    // After an abort the copies and MMAs of thread 0 may still be in flight:
    // let them land before TMEM and shared memory are released.  Thread 0
    // always committed bar_mma, so both barriers complete.
    if (tid == 0 && !ok) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar_ld, 0) && (int64_t)(globaltimer() - t0) < kDrainNs) {
        }
        while (!mbar_try_wait(bar_mma, 0) && (int64_t)(globaltimer() - t0) < kDrainNs) {
        }
    }
    tc_fence_before();
    __syncthreads();
    for (int k = tid; k < C; k += 128) hist[((size_t)bh * C + k) * nblk + blk] = hist_s[k];
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

// Exclusive scan of hist[bh] in (cluster, block) order -> offs; cluster ranges.
__global__ void __launch_bounds__(1024) km_scan(const int32_t* __restrict__ hist, int32_t* __restrict__ offs,
                                                int32_t* __restrict__ cstart, int32_t* __restrict__ ccount,
                                                KmState* __restrict__ state, int N, int C, int nblk, int it,
                                                const int* __restrict__ status) {
    __shared__ int s_part[1024];
    __shared__ int s_skip;
    if (ctl_failed(status)) return;
    const int bh = blockIdx.x, tid = threadIdx.x;
    if (tid == 0) {
        int skip = state[bh].done;
        if (!skip && it > 0 && state[bh].changed == 0) {
            state[bh].done = 1;  // labels repeat the previous pass: perm is final
            skip = 1;
        }
        if (!skip) state[bh].changed = 0;
        s_skip = skip;
    }
    __syncthreads();
    if (s_skip) return;
    const int64_t L = (int64_t)C * nblk;
    const int64_t per = (L + 1023) / 1024;
    const int64_t a = imin64(L, per * tid), b = imin64(L, a + per);
    const int32_t* hh = hist + (size_t)bh * L;
    int32_t* oo = offs + (size_t)bh * L;
    int s = 0;
    for (int64_t i = a; i < b; ++i) s += hh[i];
    s_part[tid] = s;
    __syncthreads();
    for (int d = 1; d < 1024; d <<= 1) {
        const int v = tid >= d ? s_part[tid - d] : 0;
        __syncthreads();
        s_part[tid] += v;
        __syncthreads();
    }
    int run = s_part[tid] - s;  // exclusive prefix of this segment
    for (int64_t i = a; i < b; ++i) {
        oo[i] = run;
        run += hh[i];
    }
    __syncthreads();
    for (int k = tid; k < C; k += 1024) {
        const int st = oo[(int64_t)k * nblk];
        const int en = k + 1 < C ? oo[(int64_t)(k + 1) * nblk] : N;
        cstart[(size_t)bh * C + k] = st;
        ccount[(size_t)bh * C + k] = en - st;
    }
}

__global__ void __launch_bounds__(KM_TOK) km_scatter(const int32_t* __restrict__ labels,
                                                     const int32_t* __restrict__ offs, int32_t* __restrict__ perm,
                                                     const KmState* __restrict__ state, int N, int C,
                                                     const int* __restrict__ status) {
    __shared__ int lab_s[KM_TOK];
    const int bh = blockIdx.y, blk = blockIdx.x, nblk = gridDim.x, r = threadIdx.x;
    if (ctl_failed(status) || state[bh].done) return;
    const int j = blk * KM_TOK + r;
    const int L = j < N ? labels[(size_t)bh * N + j] : -1;
    lab_s[r] = L;
    __syncthreads();
    if (j >= N) return;
    int rank = 0;
    for (int q = 0; q < r; ++q) rank += (lab_s[q] == L);
    perm[(size_t)bh * N + offs[((size_t)bh * C + L) * nblk + blk] + rank] = j;
}

constexpr int KM_SLICES = 8;

template <int D>
__global__ void __launch_bounds__(128) km_update(const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ perm,
                                                 const int32_t* __restrict__ cstart,
                                                 const int32_t* __restrict__ ccount, double* __restrict__ sums,
                                                 const KmState* __restrict__ state, int N, int C,
                                                 const int* __restrict__ status) {
    const int k = blockIdx.x, sl = blockIdx.y, bh = blockIdx.z;
    if (ctl_failed(status) || state[bh].done) return;
    const int cnt = ccount[(size_t)bh * C + k];
    if (cnt == 0) return;
    const int st = cstart[(size_t)bh * C + k];
    const int a = st + (int)(((int64_t)cnt * sl) / KM_SLICES);
    const int b = st + (int)(((int64_t)cnt * (sl + 1)) / KM_SLICES);
    constexpr int RG = 128 / D;
    const int c = threadIdx.x % D, rg = threadIdx.x / D;
    double acc = 0.0;
    const int32_t* pp = perm + (size_t)bh * N;
    const __nv_bfloat16* vb = V + (size_t)bh * N * D;
    for (int i = a + rg; i < b; i += RG) acc += (double)bf2f(vb[(size_t)pp[i] * D + c]);
    if (b > a) atomicAdd(&sums[((size_t)bh * C + k) * D + c], acc);
}

__global__ void km_finalize(__nv_bfloat16* __restrict__ c_hi, __nv_bfloat16* __restrict__ c_lo,
                            float* __restrict__ cnorm, double* __restrict__ cent64, double* __restrict__ sums,
                            const int32_t* __restrict__ ccount, const KmState* __restrict__ state, int C, int Cp,
                            int D, const int* __restrict__ status) {
    __shared__ float red[4];
    const int k = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
    if (ctl_failed(status) || state[bh].done) return;
    const int cnt = ccount[(size_t)bh * C + k];
    if (cnt == 0) return;  // an empty cluster keeps its centroid (sums are still 0)
    double* sp = &sums[((size_t)bh * C + k) * D + c];
    const double mean = *sp / (double)cnt;  // the fp64 member mean (the sum of bf16 values is exact)
    *sp = 0.0;
    cent64[((size_t)bh * C + k) * D + c] = mean;
    const size_t row = ((size_t)bh * Cp + k) * D + c;
    const __nv_bfloat16 h = __double2bfloat16(mean);
    c_hi[row] = h;
    c_lo[row] = __double2bfloat16(mean - (double)__bfloat162float(h));
    const float x = (float)mean;
    const float nrm = block_sum_d(x * x, red);
    if (c == 0) cnorm[(size_t)bh * Cp + k] = nrm;
}

// ------------------------------------------------------------------ block quantisation
// One CTA per (block of BK regrouped tokens, head).  K: amax over the block,
// inv = 448/amax, code = E4M3(k * inv), k_scale = amax/448.  V: block mean
// (fp64 sum / valid, rounded to fp32; zero when smooth == 0), residual channel
// amax folded into vamax with an integer max on the fp32 bits (all >= 0).
template <int D, int BK>
__global__ void __launch_bounds__(128) prep_kv_block(const __nv_bfloat16* __restrict__ K,
                                                     const __nv_bfloat16* __restrict__ V,
                                                     const int32_t* __restrict__ perm, int smooth,
                                                     uint8_t* __restrict__ k_fp8, float* __restrict__ k_scale,
                                                     float* __restrict__ v_mean, uint32_t* __restrict__ vamax, int N,
                                                     int T, const int* __restrict__ status) {
    constexpr int RG = 128 / D;  // row groups
    __shared__ int tok_s[BK];
    __shared__ double vsum_s[RG][D];
    __shared__ float kmax_s[128];
    __shared__ float vmax_s[RG][D];
    if (ctl_failed(status)) return;  // perm is undefined
    const int b = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int c = tid % D, rg = tid / D;
    const int valid = min(BK, N - b * BK);
    for (int r = tid; r < BK; r += 128) tok_s[r] = r < valid ? perm[(size_t)bh * N + b * BK + r] : 0;
    __syncthreads();
    const __nv_bfloat16* kb = K + (size_t)bh * N * D + c;
    const __nv_bfloat16* vb = V + (size_t)bh * N * D + c;
    float kmax = 0.0f;
    double vsum = 0.0;
    for (int r = rg; r < valid; r += RG) {
        const size_t row = (size_t)tok_s[r] * D;
        kmax = fmaxf(kmax, fabsf(bf2f(kb[row])));
        vsum += (double)bf2f(vb[row]);
    }
    kmax_s[tid] = kmax;
    vsum_s[rg][c] = vsum;
    __syncthreads();
    for (int s = 64; s > 0; s >>= 1) {
        if (tid < s) kmax_s[tid] = fmaxf(kmax_s[tid], kmax_s[tid + s]);
        __syncthreads();
    }
    const float amax = kmax_s[0];
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
    if (tid == 0) k_scale[(size_t)bh * T + b] = __fdiv_rn(amax, 448.0f);
    double tot = 0.0;
#pragma unroll
    for (int q = 0; q < RG; ++q) tot += vsum_s[q][c];
    const float mu = smooth ? (float)(tot / (double)valid) : 0.0f;
    if (rg == 0) v_mean[((size_t)bh * T + b) * D + c] = mu;
    uint8_t* kout = k_fp8 + ((size_t)bh * T * BK + (size_t)b * BK) * D;
    float vmax = 0.0f;
    for (int r = rg; r < BK; r += RG) {
        uint8_t code = 0;
        if (r < valid) {
            const size_t row = (size_t)tok_s[r] * D;  // second read of the gathered rows hits L2
            code = (uint8_t)(e4m3x2(__fmul_rn(bf2f(kb[row]), inv), 0.0f) & 0xFF);
            vmax = fmaxf(vmax, fabsf(__fsub_rn(bf2f(vb[row]), mu)));
        }
        kout[(size_t)r * D + c] = code;
    }
    vmax_s[rg][c] = vmax;
    __syncthreads();
    if (rg == 0) {
        float m = vmax_s[0][c];
#pragma unroll
        for (int q = 1; q < RG; ++q) m = fmaxf(m, vmax_s[q][c]);
        atomicMax(&vamax[(size_t)bh * D + c], __float_as_uint(m));
    }
}

// V-Smooth off: identity order, every token in cluster 0.
__global__ void identity_order(int32_t* __restrict__ perm, int32_t* __restrict__ labels, int64_t total, int N) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        perm[i] = (int32_t)(i % N);
        labels[i] = 0;
    }
}

// E4M3 residual with per-channel scales, written transposed: vt[bh][c][token].
template <int D, int BK>
__global__ void __launch_bounds__(128) prep_v_quant(const __nv_bfloat16* __restrict__ V,
                                                    const int32_t* __restrict__ perm, int smooth,
                                                    const float* __restrict__ v_mean,
                                                    const uint32_t* __restrict__ vamax, uint8_t* __restrict__ vt_fp8,
                                                    float* __restrict__ v_scale, int N, int T,
                                                    const int* __restrict__ status) {
    constexpr int RG = 128 / D;
    constexpr int STRIDE = BK + 4;  // bytes per channel row in smem (conflict-free word stores)
    __shared__ int tok_s[BK];
    __shared__ uint32_t cs[D * STRIDE / 4];
    if (ctl_failed(status)) return;  // perm is undefined
    const int b = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int c = tid % D, rg = tid / D;
    const int valid = min(BK, N - b * BK);
    const int Tp = T * BK;
    for (int r = tid; r < BK; r += 128) tok_s[r] = r < valid ? perm[(size_t)bh * N + b * BK + r] : 0;
    const float amax = __uint_as_float(vamax[(size_t)bh * D + c]);
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
    if (b == 0 && rg == 0) v_scale[(size_t)bh * D + c] = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const float mu = v_mean[((size_t)bh * T + b) * D + c];
    __syncthreads();
    for (int r4 = rg; r4 < BK / 4; r4 += RG) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = 4 * r4 + e;
            x[e] = 0.0f;
            if (r < valid) {
                const float v = bf2f(V[((size_t)bh * N + tok_s[r]) * D + c]);
                x[e] = __fmul_rn(__fsub_rn(v, mu), inv);
            }
        }
        const uint32_t w = (uint32_t)e4m3x2(x[0], x[1]) | ((uint32_t)e4m3x2(x[2], x[3]) << 16);
        // padding tokens must be code 0 (x = +0 encodes to 0x00)
        cs[(c * STRIDE) / 4 + r4] = w;
    }
    __syncthreads();
    constexpr int CHUNKS = BK / 16;
    for (int i = tid; i < D * CHUNKS; i += 128) {
        const int cc = i / CHUNKS, ch = i % CHUNKS;
        const uint32_t* src = cs + (cc * STRIDE) / 4 + ch * 4;
        *reinterpret_cast<uint4*>(vt_fp8 + ((size_t)bh * D + cc) * Tp + (size_t)b * BK + 16 * ch) =
            make_uint4(src[0], src[1], src[2], src[3]);
    }
}

// Per-token Q: amax over d, inv = 448/amax, code = E4M3(q * inv), sq = amax/448.
template <int D>
__global__ void __launch_bounds__(256) quant_q(const __nv_bfloat16* __restrict__ Q, uint8_t* __restrict__ q_fp8,
                                               float* __restrict__ sq, int64_t tokens) {
    constexpr int PER = D / 32;  // values per lane
    const int64_t tok = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (tok >= tokens) return;
    float x[PER];
    const __nv_bfloat16* src = Q + tok * D + lane * PER;
    if constexpr (PER == 4) {
        const uint2 raw = *reinterpret_cast<const uint2*>(src);
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = bf2f(h[e]);
    } else {
        const uint32_t raw = *reinterpret_cast<const uint32_t*>(src);
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
        for (int e = 0; e < PER; ++e) x[e] = bf2f(h[e]);
    }
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < PER; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float inv = m > 0.0f ? __fdiv_rn(448.0f, m) : 0.0f;
    if constexpr (PER == 4) {
        const uint32_t w = (uint32_t)e4m3x2(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv)) |
                           ((uint32_t)e4m3x2(__fmul_rn(x[2], inv), __fmul_rn(x[3], inv)) << 16);
        *reinterpret_cast<uint32_t*>(q_fp8 + tok * D + lane * 4) = w;
    } else {
        *reinterpret_cast<uint16_t*>(q_fp8 + tok * D + lane * 2) =
            e4m3x2(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv));
    }
    if (lane == 0) sq[tok] = __fdiv_rn(m, 448.0f);
}

__global__ void e4m3_encode_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (uint8_t)(e4m3x2(x[i], 0.0f) & 0xFF);
}

// ------------------------------------------------------------------ host launchers

template <int D>
static cudaError_t kmeans_t(const PrepLaunch& p, cudaStream_t s) {
    const int nblk = (p.N + KM_TOK - 1) / KM_TOK;
    const int Cp = (p.C + 15) & ~15;
    const size_t smem = 1024 + (size_t)KM_TOK * D * 2 + 2 * (size_t)Cp * D * 2 + 2 * 256 * 4 + 64;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(km_assign<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    CUtensorMap tv, th, tl;
    if (!make_tmap_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.V, D, p.N, p.BH, 64, KM_TOK) ||
        !make_tmap_3d(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.c_hi, D, Cp, p.BH, 64, Cp) ||
        !make_tmap_3d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.c_lo, D, Cp, p.BH, 64, Cp))
        return cudaErrorInvalidValue;
    km_init<<<dim3(Cp, p.BH), D, 0, s>>>(p.V, p.c_hi, p.c_lo, p.cnorm, p.cent64, p.sums, p.state, p.vamax, p.N, p.C,
                                         Cp, D);
    for (int it = 0; it < p.iters; ++it) {
        km_assign<D><<<dim3(nblk, p.BH), 128, smem, s>>>(tv, th, tl, p.cnorm, p.cent64, p.V, p.labels, p.hist,
                                                          p.state, p.N, p.C, Cp, it, p.ctl);
        km_scan<<<p.BH, 1024, 0, s>>>(p.hist, p.offs, p.cstart, p.ccount, p.state, p.N, p.C, nblk, it,
                                      p.ctl.status);
        km_scatter<<<dim3(nblk, p.BH), KM_TOK, 0, s>>>(p.labels, p.offs, p.perm, p.state, p.N, p.C,
                                                       p.ctl.status);
        if (it + 1 < p.iters) {
            km_update<D><<<dim3(p.C, KM_SLICES, p.BH), 128, 0, s>>>(p.V, p.perm, p.cstart, p.ccount, p.sums, p.state,
                                                                    p.N, p.C, p.ctl.status);
            km_finalize<<<dim3(p.C, p.BH), D, 0, s>>>(p.c_hi, p.c_lo, p.cnorm, p.cent64, p.sums, p.ccount, p.state,
                                                      p.C, Cp, D, p.ctl.status);
        }
    }
    return cudaGetLastError();
}

template <int D, int BK>
static cudaError_t blocks_t(const PrepLaunch& p, cudaStream_t s) {
    const int T = (p.N + BK - 1) / BK;
    if (!p.smooth) {  // plain per-channel FP8 V: identity order, zeroed channel maxima
        const int64_t total = (int64_t)p.BH * p.N;
        identity_order<<<(unsigned)imin64((total + 255) / 256, 148 * 32), 256, 0, s>>>(p.perm, p.labels,
                                                                                             total, p.N);
        cudaError_t e = cudaMemsetAsync(p.vamax, 0, sizeof(uint32_t) * (size_t)p.BH * D, s);
        if (e != cudaSuccess) return e;
    }
    prep_kv_block<D, BK><<<dim3(T, p.BH), 128, 0, s>>>(p.K, p.V, p.perm, p.smooth, p.k_fp8, p.k_scale, p.v_mean,
                                                       p.vamax, p.N, T, p.ctl.status);
    prep_v_quant<D, BK><<<dim3(T, p.BH), 128, 0, s>>>(p.V, p.perm, p.smooth, p.v_mean, p.vamax, p.vt_fp8, p.v_scale,
                                                      p.N, T, p.ctl.status);
    return cudaGetLastError();
}

cudaError_t launch_prep(const PrepLaunch& p, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    if (p.smooth) {
        e = p.D == 128 ? kmeans_t<128>(p, s) : kmeans_t<64>(p, s);
        if (e != cudaSuccess) return e;
    }
    if (p.D == 128 && p.BK == 128) return blocks_t<128, 128>(p, s);
    if (p.D == 128 && p.BK == 64) return blocks_t<128, 64>(p, s);
    if (p.D == 64 && p.BK == 128) return blocks_t<64, 128>(p, s);
    return blocks_t<64, 64>(p, s);
}

cudaError_t launch_quant_q(const __nv_bfloat16* Q, uint8_t* q_fp8, float* sq, int64_t tokens, int D,
                           cudaStream_t s) {
    const unsigned grid = (unsigned)((tokens + 7) / 8);
    if (D == 128)
        quant_q<128><<<grid, 256, 0, s>>>(Q, q_fp8, sq, tokens);
    else
        quant_q<64><<<grid, 256, 0, s>>>(Q, q_fp8, sq, tokens);
    return cudaGetLastError();
}

cudaError_t launch_e4m3_encode(const float* x, uint8_t* out, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const unsigned grid = (unsigned)imin64((n + 255) / 256, 148 * 16);
    e4m3_encode_kernel<<<grid, 256, 0, s>>>(x, out, n);
    return cudaGetLastError();
}

}  // namespace vc
