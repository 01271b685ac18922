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
//   C <= 64, per pass:
//     km_pass                 one persistent launch: labels = argmin_k |c_k|^2 - 2 v.c_k on
//                             tensor cores (ties -> lowest k), per-(cluster, 128-token tile)
//                             histogram, change count, near ties listed per CTA; the fp64
//                             member sums from the same V tile (pass 0: every token; later:
//                             the tokens whose label changed, moved between sums)
//     km_refine               the near ties decided exactly (fp32 bounds, else fp64); fixes
//                             labels, counts and sums
//     km_finalize             c_k = sum / count (empty clusters keep c_k); a head whose labels
//                             did not change is final (its later passes would repeat)
//   then once: km_scan, km_scatter (the stable regroup from the last labels)
//   C > 64, per pass: km_assign (the assignment alone), km_refine, km_scan (the head's
//     final check), km_scatter, km_update (fp64 sums over slices of the stable order),
//     km_finalize
//   identity_order            V-Smooth off (smooth 0): perm = identity, labels 0, no k-means
//   (smooth 2 runs no k-means kernel and keeps the perm already in the prep buffers)
//   prep_kv_block             per block: K amax scale + E4M3 K, V block mean (fp64 sum),
//                             residual channel amax
//   prep_v_quant              per-channel residual scale, E4M3 residual, transposed
//   prep_v_quant_nvfp4        the same with the 4-bit (NVFP4) residual and its block scales
//   quant_q                   per-token E4M3 Q (used by the attention call)
#include <math.h>

#include "vc_launch.cuh"

namespace vc {

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// 16 bytes from global to shared memory without passing through registers
// (both addresses 16-byte aligned), so a thread keeps all its pieces of a
// gather in flight at once; cp_async_wait_all makes the thread's own copies
// complete and visible to it (other threads need a barrier after).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------------ k-means
// Centroids live as bf16 hi/lo pairs, row-major [BH, Cp, D] (Cp = C rounded up
// to 16; pad rows are zero), plus fp32 squared norms [BH, Cp]: v.c is computed
// on tensor cores as v.hi + v.lo (v is exact in bf16), so the distance
// |c|^2 - 2 v.c carries about 2^-16 relative error in c.

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
                        double* __restrict__ sums, KmState* __restrict__ state, uint32_t* __restrict__ vamax,
                        int* __restrict__ tie_count, int N,
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
    if (k == 0 && bh == 0 && c < 2) tie_count[c] = 0;
    if (k == 0) {
        vamax[(size_t)bh * D + c] = 0u;
        if (c == 0) state[bh] = KmState{{0, 0}, 0, 0};
    }
}

constexpr int KM_TOK = 128;  // tokens per tile (the MMA's M)

// Shared-memory plan of km_assign, from a 1024-byte aligned base:
//   V tile x2 | centroid hi | centroid lo | |c|^2 | histograms x2 | scratch | barriers
struct KmLayout {
    uint32_t v_bytes, c_bytes, off_v, off_chi, off_clo, off_cn, off_hist, off_red, off_bar, off_misc, bytes;
    __host__ __device__ KmLayout(int D, int Cp) {
        v_bytes = KM_TOK * D * 2;
        c_bytes = Cp * D * 2;
        off_v = 0;
        off_chi = v_bytes;  // one V tile: the next is loaded while the CUDA cores work
        off_clo = off_chi + c_bytes;
        off_cn = off_clo + c_bytes;            // [256] |c_k|^2
        off_hist = off_cn + 256 * 4;           // [2][256] per-tile cluster counts
        off_red = off_hist + 2 * 256 * 4;
        off_bar = off_red + 64;
        off_misc = off_bar + 64;
        bytes = off_misc + 16 + 1024;  // + alignment slack
    }
};

// Assignment pass on tensor cores.  One CTA takes `tpc` consecutive 128-token
// tiles of one head; the centroids are loaded once, the V tiles stream through
// a double buffer, and the MMA of tile j+1 runs while the CUDA cores finish
// tile j:
//   S[token, k] = v . c_hi + v . c_lo   (kind::f16, bf16 x bf16 -> fp32 in TMEM)
//   label = argmin_k (|c_k|^2 - 2 S[token, k]), ties to the lowest k,
// with near-ties decided again in fp64.  Per tile: labels, the per-cluster
// histogram of the tile (for the stable regroup) and the change count.
template <int D>
__global__ void __launch_bounds__(128, 3) km_assign(const __grid_constant__ CUtensorMap tm_v,
                                                 const __grid_constant__ CUtensorMap tm_chi,
                                                 const __grid_constant__ CUtensorMap tm_clo,
                                                 const float* __restrict__ cnorm, const double* __restrict__ cent64,
                                                 const __nv_bfloat16* __restrict__ V, float* __restrict__ vnorm2,
                                                 int32_t* __restrict__ labels, int32_t* __restrict__ hist,
                                                 KmTie* __restrict__ ties, int* __restrict__ tie_count,
                                                 KmState* __restrict__ state, int N, int C, int Cp, int it, int tpc,
                                                 DevCtl ctl) {
    const int bh = blockIdx.y, nblk = (N + KM_TOK - 1) / KM_TOK;
    const int blk0 = blockIdx.x * tpc;
    const int nt = min(tpc, nblk - blk0);
    // both uniform over the CTA, before any barrier or TMEM use
    if (ctl_failed(ctl.status) || state[bh].done || nt <= 0) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const KmLayout L(D, Cp);
    float* cn_s = reinterpret_cast<float*>(smem + L.off_cn);
    int* hist_s = reinterpret_cast<int*>(smem + L.off_hist);  // [2][256]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.off_misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.off_misc + 4);
    const uint32_t bar_c = base + L.off_bar, bar_v0 = bar_c + 8, bar_mma0 = bar_c + 24;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t ncols = 2 * Cp <= 32 ? 32 : (2 * Cp <= 64 ? 64 : (2 * Cp <= 128 ? 128 : (2 * Cp <= 256 ? 256 : 512)));

    if (tid == 0) {
        mbar_init(bar_c, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_v0 + 8 * i, 1);
            mbar_init(bar_mma0 + 8 * i, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), ncols);
        tmem_relinquish();
    }
    // |c_k|^2 (pad clusters +inf, never chosen) and max_k |c_k|^2 of the head
    uint32_t* red_s = reinterpret_cast<uint32_t*>(smem + L.off_red);
    uint32_t cmax_bits = 0;
    for (int k = tid; k < Cp; k += 128) {
        const float x = k < C ? cnorm[(size_t)bh * Cp + k] : INFINITY;
        cn_s[k] = x;
        if (k < C) cmax_bits = max(cmax_bits, __float_as_uint(x));  // x >= 0: bit order is value order
    }
    cmax_bits = __reduce_max_sync(0xffffffffu, cmax_bits);
    if (lane == 0) red_s[warp] = cmax_bits;
    for (int k = tid; k < 2 * 256; k += 128) hist_s[k] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const float cmax_r = sqrtf(__uint_as_float(max(max(red_s[0], red_s[1]), max(red_s[2], red_s[3]))));

    const uint32_t sV = base + L.off_v, sCh = base + L.off_chi, sCl = base + L.off_clo;
    auto load_v = [&](int j) {  // thread 0; tile j completes phase j & 1 of bar_v0
        mbar_expect_tx_arrive(bar_v0, L.v_bytes);
#pragma unroll
        for (int kc = 0; kc < D / 64; ++kc)
            tma_load_3d(sV + kc * (KM_TOK * 128), &tm_v, bar_v0, 64 * kc, (blk0 + j) * KM_TOK, bh);
    };
    const uint32_t idesc = idesc_bf16_f32(Cp);
    auto issue_mma = [&](int j) {  // thread 0, after V tile j (and the centroids) landed
        const uint32_t b = j & 1;
        const uint32_t sA = sV, acc = tmem + b * Cp;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_bf16(acc, smem_desc(sA + (kk >> 2) * (KM_TOK * 128) + off, 128),
                     smem_desc(sCh + (kk >> 2) * (Cp * 128) + off, 128), idesc, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_bf16(acc, smem_desc(sA + (kk >> 2) * (KM_TOK * 128) + off, 128),
                     smem_desc(sCl + (kk >> 2) * (Cp * 128) + off, 128), idesc, 1u);
        }
        mma_commit(bar_mma0 + 8 * b);
    };

    int v_issued = 0, mma_issued = 0;  // thread 0's in-flight bookkeeping
    bool ok = true;
    if (tid == 0) {
        mbar_expect_tx_arrive(bar_c, 2 * L.c_bytes);
#pragma unroll
        for (int kc = 0; kc < D / 64; ++kc) {
            tma_load_3d(sCh + kc * (Cp * 128), &tm_chi, bar_c, 64 * kc, 0, bh);
            tma_load_3d(sCl + kc * (Cp * 128), &tm_clo, bar_c, 64 * kc, 0, bh);
        }
        load_v(0);
        v_issued = 1;
        ok = mbar_wait(bar_c, 0, ctl, abort_flag) && mbar_wait(bar_v0, 0, ctl, abort_flag);
        if (ok) {
            issue_mma(0);
            mma_issued = 1;
        }
    }
    int changed = 0;
    for (int j = 0; j < nt; ++j) {
        const int b = j & 1;
        const int n0 = (blk0 + j) * KM_TOK;
        if (j >= 1) {  // the previous tile's histogram is complete (barrier below)
            int* hp = hist_s + (b ^ 1) * 256;
            for (int k = tid; k < C; k += 128) {
                hist[((size_t)bh * C + k) * nblk + blk0 + j - 1] = hp[k];
                hp[k] = 0;
            }
        }
        bool okj = __all_sync(0xffffffffu, ok && mbar_wait(bar_mma0 + 8 * b, (j >> 1) & 1, ctl, abort_flag));
        tc_fence_after();
        const int n = n0 + tid;
        const bool valid = n < N;
        float vn2 = 0.0f;
        if (it == 0) {  // |v|^2 once per prep, from the V tile before it is overwritten
            if (okj) {
                const uint8_t* arow = smem + L.off_v + tid * 128;
#pragma unroll
                for (int kc = 0; kc < D / 64; ++kc)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 raw =
                            *reinterpret_cast<const uint4*>(arow + kc * (KM_TOK * 128) + ((ch ^ (tid & 7)) << 4));
                        const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                        for (int e = 0; e < 8; ++e) vn2 = fmaf(bf2f(hv[e]), bf2f(hv[e]), vn2);
                    }
                if (valid) vnorm2[(size_t)bh * N + n] = vn2;
            }
            __syncthreads();
        } else if (okj && valid) {
            vn2 = vnorm2[(size_t)bh * N + n];
        }
        if (tid == 0 && okj && j + 1 < nt) {  // MMA j has read the V tile
            load_v(j + 1);
            v_issued = j + 2;
        }
        if (okj) {
            const uint32_t lane_tmem = tmem + b * Cp + ((uint32_t)(warp * 32) << 16);
            // Pass 1: best and runner-up of the tensor-core distances
            // d_k = |c_k|^2 - 2 v.c_k.  With Cp <= 64 the distances stay in
            // registers for the near-tie masks below.
            float b4[4] = {INFINITY, INFINITY, INFINITY, INFINITY}, s4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
            int k4[4] = {0, 0, 0, 0};  // four independent chains: candidate k goes to chain k % 4
            float dk[64];
            for (int g = 0; g < Cp; g += 64) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (g + 16 * q < Cp) tmem_ld16(lane_tmem + g + 16 * q, dk + 16 * q);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 16; ++q4) {
                    if (g + 4 * q4 < Cp) {
                        const float4 cn = reinterpret_cast<const float4*>(cn_s + g)[q4];
                        const float cv[4] = {cn.x, cn.y, cn.z, cn.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float d = fmaf(-2.0f, dk[4 * q4 + e], cv[e]);
                            dk[4 * q4 + e] = d;
                            const bool lt = d < b4[e];
                            s4[e] = fminf(s4[e], fmaxf(b4[e], d));
                            b4[e] = fminf(b4[e], d);
                            k4[e] = lt ? g + 4 * q4 + e : k4[e];
                        }
                    }
                }
            }
            // merge the chains: best (ties to the lowest k) and runner-up
            float best = b4[0], second = s4[0];
            int bestk = k4[0];
#pragma unroll
            for (int e = 1; e < 4; ++e) {
                second = fminf(fminf(second, s4[e]), fmaxf(best, b4[e]));
                if (b4[e] < best || (b4[e] == best && k4[e] < bestk)) {
                    best = b4[e];
                    bestk = k4[e];
                }
            }
            // Error bound of the tensor-core distance d = |c|^2 - 2 v.c: the bf16
            // hi/lo centroid carries 2^-16 relative error per channel, the
            // products are exact, and the fp32 accumulation of the 2 D products
            // errs by at most 2^-15 of sum |v_c c_c| (one unit of fp32
            // truncation per addition), so 2 v.c errs by at most
            // 3 * 2^-15 |v||c| <= 2^-15.4 (|v| + max|c|)^2; |c|^2 in fp32 adds
            // far less.  If every d errs by at most E, the fp64 argmin lies
            // within 2E of the tensor-core best, so the clusters within
            // 2^-13 (|v| + max|c|)^2 of the best (2.6 times 2E) are decided
            // again in fp64 from the fp64 centroids, as the Lloyd step defines
            // the distance (sum over channels of (v - c)^2).
            const float rad = sqrtf(vn2) + cmax_r;
            const float margin = ldexpf(rad * rad, -13);
            const bool refine = valid && C > 1 && (second - best) <= margin;
            // Near ties go to the list that km_refine decides in fp64; the
            // label written now is the tensor-core choice.
            const int32_t old_label = valid && it > 0 ? labels[(size_t)bh * N + n] : -1;
            const uint32_t rmask = __ballot_sync(0xffffffffu, refine);
            if (rmask != 0) {
                int first = 0;
                if (lane == 0) first = atomicAdd(tie_count + (it & 1), __popc(rmask));
                first = __shfl_sync(0xffffffffu, first, 0);
                KmTie* e = ties + first + __popc(rmask & ((1u << lane) - 1));
                const float lim = best + margin;
                for (int g = 0; g < Cp; g += 64) {
                    if (Cp > 64) {  // the group's distances again, from TMEM
#pragma unroll
                        for (int q = 0; q < 4; ++q)  // warp-collective: every lane loads
                            if (g + 16 * q < Cp) tmem_ld16(lane_tmem + g + 16 * q, dk + 16 * q);
                        tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 64; ++jj)
                            if (g + jj < Cp) dk[jj] = fmaf(-2.0f, dk[jj], cn_s[g + jj]);
                    }
                    if (refine) {
                        uint32_t m0 = 0, m1 = 0;  // candidates g..g+31 and g+32..g+63
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            if (g + jj < Cp && dk[jj] <= lim) m0 |= 1u << jj;
                            if (g + 32 + jj < Cp && dk[32 + jj] <= lim) m1 |= 1u << jj;
                        }
                        e->mask[g >> 5] = m0;
                        if ((g >> 5) + 1 < 8) e->mask[(g >> 5) + 1] = m1;
                    }
                }
                if (refine) *reinterpret_cast<int4*>(e) = make_int4(bh, n, old_label, bestk);
            }
            const int label = bestk;
            if (valid) {
                if (it == 0 || old_label != label) ++changed;
                labels[(size_t)bh * N + n] = label;
                atomicAdd(&hist_s[b * 256 + label], 1);
            }
        }
        if (tid == 0 && ok && okj && j + 1 < nt) {
            // MMA j+1 into the other accumulator (read out by tile j-1) while
            // the other warps finish tile j
            ok = mbar_wait(bar_v0, (j + 1) & 1, ctl, abort_flag);
            if (ok) {
                issue_mma(j + 1);
                mma_issued = j + 2;
            }
        }
        tc_fence_before();
        ok = __syncthreads_and(okj && ok) != 0;  // also frees accumulator b and histogram b^1
        if (!ok) break;
    }
    if (ok) {
        const int j = nt - 1;
        const int* hp = hist_s + (j & 1) * 256;
        for (int k = tid; k < C; k += 128) hist[((size_t)bh * C + k) * nblk + blk0 + j] = hp[k];
    }
    changed = __reduce_add_sync(0xffffffffu, changed);
    if (lane == 0 && changed) atomicAdd(&state[bh].chg[it & 1], changed);
    // After an abort thread 0's last copies and MMAs may still be in flight:
    // let them land before shared memory and TMEM are released.
    if (tid == 0 && !ok) {
        const uint64_t t0 = globaltimer();
        auto drain = [&](uint32_t bar, uint32_t parity) {
            while (!mbar_try_wait(bar, parity) && (int64_t)(globaltimer() - t0) < kDrainNs) {
            }
        };
        drain(bar_c, 0);
        if (v_issued > 0) drain(bar_v0, (v_issued - 1) & 1);  // earlier tiles landed before the next was issued
        for (int t = max(0, mma_issued - 2); t < mma_issued; ++t) drain(bar_mma0 + 8 * (t & 1), (t >> 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

// ------------------------------------------------------------------ fused pass
// One k-means pass for C <= 64, persistent: one CTA per SM takes an equal,
// contiguous share of the (head, 128-token tile) units of the heads whose
// labels still change, and reads each V tile once for both halves of the
// Lloyd step:
//   assignment  label = argmin_k |c_k|^2 - 2 v.c_k on tensor cores (kind::f16,
//               v . c_hi + v . c_lo in TMEM), ties to the lowest k, near ties
//               listed for km_refine, the tile's cluster histogram, and the
//               tile's tokens grouped by cluster (a counting sort);
//   update      the member sums from the same V tile in shared memory: each
//               update warp owns a contiguous range of clusters, whose tokens
//               are one contiguous block of the grouped tile; it walks the block four
//               tokens at a time, adds each run of a cluster in registers and
//               the run's sum to the CTA's fp64 sums in shared memory; those go
//               to the head's global sums
//               (one fp64 atomic each) when the CTA leaves the head.  Every
//               fp64 addition of bf16 values is exact (for values of typical
//               range), so the sums do not depend on the order and equal the
//               oracle's sequential ones.  Loops stay short: with four warp
//               roles in one CTA, long unrolled code stalls on instruction
//               fetch.
// `mode` 1 is that full accumulation (the sums start from zero).  Mode 3 keeps
// the sums and has the update warps move only the tokens whose label changed:
// the tile's changed tokens grouped by new cluster are added, grouped by old
// cluster subtracted (for pass 1, where most labels still hold).  Mode 2 keeps
// the sums of the previous pass and moves only the tokens whose label changed
// (the assignment warps subtract the row from the old cluster's global sums
// and add it to the new one's, fp64 atomics): exact like a fresh sum, and
// cheap once few labels change.  Mode 0 (the last pass) writes labels and
// histograms only.
// Warps: 0 TMA producer (V tiles through a ring of stages; a head's centroids
// when the CTA enters it), 1 MMA issuer (tile i into TMEM accumulator
// i % kAcc), then G assignment groups of four warps (group g takes the CTA's
// tiles i = g mod G; a thread per token), then U update warps (D/32 channels a
// lane; warp u owns clusters (64/U)u onwards).  Shapes: passes 0 and 1 (sum
// every token; move a seventh of them) 1 group and 8 update warps (2 groups
// and 4 measured slower for pass 1); later passes (move a few per mille by
// atomics) 3 groups and none.
constexpr int KP_SEG = 68;  // per stage: 65 cluster offsets, padded
constexpr int KP_MAX_GRID = kKmTieRegions;  // near-tie regions the workspace holds

template <int G, int U>
struct KpShape {
    static constexpr int kGroups = G;
    static constexpr int kUpd = U;                  // update warps
    static constexpr int kCpw = U > 0 ? 64 / U : 0;  // clusters a update warp owns
    static constexpr int kStages = U > 0 ? 3 : 4;
    static constexpr int kAcc = G < 2 ? 2 : G;  // TMEM accumulators
    static constexpr int kThreads = 32 * (2 + 4 * G + kUpd);
};

// Shared-memory plan of km_pass, from a 1024-byte aligned base:
//   V ring | centroid hi | centroid lo | fp64 sums [64][D] | |c|^2 per group |
//   tile order and its labels per stage | cluster offsets per stage | label
//   counts per group x2 | scratch | barriers
struct KpLayout {
    uint32_t v_bytes, c_bytes, off_v, off_chi, off_clo, off_sum, off_cn, off_ord, off_slab, off_seg, off_ord2,
        off_slab2, off_seg2, off_cnt, off_misc, off_bar, bytes;
    __host__ __device__ KpLayout(int D, int Cp, int S, int G, int nacc, bool with_sums) {
        v_bytes = KM_TOK * D * 2;
        c_bytes = Cp * D * 2;
        off_v = 0;
        off_chi = off_v + S * v_bytes;
        off_clo = off_chi + c_bytes;
        off_sum = off_clo + c_bytes;                      // [64][D] double (the shape with update warps)
        off_cn = off_sum + (with_sums ? 64 * D * 8 : 0);  // [G][64] float, then [G] max |c|^2 bits
        off_ord = off_cn + ((G * 65 * 4 + 15) & ~15);     // [stage][128] tile rows grouped by cluster
        off_slab = off_ord + S * KM_TOK;                  // [stage][128] their clusters
        off_seg = off_slab + S * KM_TOK;                  // [stage][KP_SEG] first grouped position of each cluster
        off_ord2 = off_seg + S * KP_SEG * 4;              // the same for the subtract list of mode 3
        off_slab2 = off_ord2 + S * KM_TOK;
        off_seg2 = off_slab2 + S * KM_TOK;
        off_cnt = off_seg2 + S * KP_SEG * 4;              // [G][2][3][64] label counts of a group's tile
        off_misc = off_cnt + G * 2 * 3 * 64 * 4;          // [16] ints, see km_pass
        off_bar = off_misc + 64;
        bytes = off_bar + 8 * (3 * S + 2 * nacc + 3) + 1024;  // + alignment slack
    }
};

// All-of over the threads of named barrier `id` (bar.red.and): every thread
// gets the same answer, so a decision taken on it is uniform.
__device__ __forceinline__ bool named_barrier_and(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// The walk over a CTA's units: (bh, tile) in head-major order over the heads
// not yet final.
struct KpWalk {
    int bh, tile;
    __device__ __forceinline__ void next(const KmState* state, int BH, int nblk) {
        if (++tile == nblk) {
            tile = 0;
            do {
                ++bh;
            } while (bh < BH && state[bh].done);
        }
    }
};

// bf16 -> fp64 by placing the bits: a bf16 with sign s, exponent e and
// mantissa m read as the fp64 with sign s, exponent field e and mantissa m
// (top bits) is the bf16 value times 2^-896, exactly, for every finite bf16
// (normal: 2^(e-1023) (1 + m/128) = 2^-896 * 2^(e-127) (1 + m/128); zero and
// subnormal: m 2^-1029 = 2^-896 * m 2^-133).  Sums of these scaled values are
// exact whenever the unscaled ones are; multiplying by 2^896 (kBf16Unscale)
// gives the sum back exactly.  The high word is the bf16's 16 bits moved to
// the top of a 32-bit word, shifted right by 3 with the sign copied, and the
// copies of the sign and the bits shifted in from below cleared.
constexpr double kBf16Unscale = 0x1p896;
__device__ __forceinline__ double bf16hi_scaled(uint32_t w) {  // bits 16..31 of w
    return __hiloint2double((int)(((int)w >> 3) & 0x8FFFE000), 0);
}
__device__ __forceinline__ double bf16lo_scaled(uint32_t w) {  // bits 0..15 of w
    return bf16hi_scaled(w << 16);
}

template <int D, int G, int U>
__global__ void __launch_bounds__(KpShape<G, U>::kThreads, 1)
    km_pass(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_chi,
            const __grid_constant__ CUtensorMap tm_clo, const float* __restrict__ cnorm, float* __restrict__ vnorm2,
            int32_t* __restrict__ labels, int32_t* __restrict__ hist, double* __restrict__ sums,
            KmTie* __restrict__ ties, int* __restrict__ tie_regions, KmState* __restrict__ state, int BH, int N,
            int C, int Cp, int it, int mode, DevCtl ctl) {
    using Shape = KpShape<G, U>;
    constexpr bool UPD = U > 0;
    constexpr int CPW = Shape::kCpw;
    constexpr int S = Shape::kStages, NACC = Shape::kAcc, ASG = 4 * G;
    const bool accumulate = UPD && (mode == 1 || mode == 3);
    if (ctl_failed(ctl.status)) return;
    const int nblk = (N + KM_TOK - 1) / KM_TOK;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_base);
    const KpLayout L(D, Cp, S, G, NACC, UPD);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // scratch: [0] TMEM base, [1] abort flag, [4] units, [5] first head,
    // [6] first tile, [7] near ties listed, [8] near-tie region start
    int* misc = reinterpret_cast<int*>(smem + L.off_misc);
    volatile int* abort_flag = misc + 1;
    int* tie_s = misc + 7;
    int* cnt_s = reinterpret_cast<int*>(smem + L.off_cnt);
    const uint32_t bar0 = base + L.off_bar;
    auto b_vfull = [&](int st) { return bar0 + 8u * st; };
    auto b_vempty = [&](int st) { return bar0 + 8u * (S + st); };
    auto b_lfull = [&](int st) { return bar0 + 8u * (2 * S + st); };
    auto b_accfull = [&](int b) { return bar0 + 8u * (3 * S + b); };
    auto b_accempty = [&](int b) { return bar0 + 8u * (3 * S + NACC + b); };
    const uint32_t b_cfull = bar0 + 8u * (3 * S + 2 * NACC), b_cempty = b_cfull + 8, b_mmadone = b_cfull + 16;
    if (tid == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(b_vfull(st), 1);
            // the MMA warp's commit, the 4 warps of the assignment group, the update warps
            mbar_init(b_vempty(st), 1 + 4 + (accumulate ? Shape::kUpd : 0));
            mbar_init(b_lfull(st), 4);
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(b_accfull(b), 1);
            mbar_init(b_accempty(b), 4);
        }
        mbar_init(b_cfull, 1);
        mbar_init(b_cempty, 1);
        mbar_init(b_mmadone, 1);
        *abort_flag = 0;
        *tie_s = 0;
        fence_mbar_init();
    }
    for (int i = tid; i < G * 2 * 3 * 64; i += blockDim.x) cnt_s[i] = 0;
    double* sums_s = reinterpret_cast<double*>(smem + L.off_sum);
    if (accumulate)
        for (int i = tid; i < 64 * D; i += blockDim.x) sums_s[i] = 0.0;
    const uint32_t ncols = NACC * Cp <= 32 ? 32 : (NACC * Cp <= 64 ? 64 : (NACC * Cp <= 128 ? 128 : 256));
    if (warp == 1) {
        tmem_alloc(smem_u32(reinterpret_cast<uint32_t*>(misc)), ncols);
        tmem_relinquish();
    }
    if (warp == 2) {
        // This CTA's share of the live units: the heads still changing, nblk
        // units each, split evenly over the grid.
        int live = 0;
        for (int bh = lane; bh < BH; bh += 32) live += state[bh].done == 0;
        live = __reduce_add_sync(0xffffffffu, live);
        const int64_t units = (int64_t)live * nblk;
        const int64_t lu0 = units * blockIdx.x / gridDim.x, lu1 = units * (blockIdx.x + 1) / gridDim.x;
        // the head of live unit lu0: the (lu0 / nblk)-th live head
        const int64_t target = lu0 / nblk;
        int seen = 0, bh0 = BH;
        for (int b0 = 0; b0 < BH && lu1 > lu0; b0 += 32) {
            const int bh = b0 + lane;
            uint32_t m = __ballot_sync(0xffffffffu, bh < BH && state[bh].done == 0);
            if (seen + __popc(m) > target) {
                for (int q = 0; q < (int)(target - seen); ++q) m &= m - 1;
                bh0 = b0 + __ffs(m) - 1;
                break;
            }
            seen += __popc(m);
        }
        if (lane == 0) {
            misc[4] = (int)(lu1 - lu0);
            misc[5] = bh0;
            misc[6] = (int)(lu0 % nblk);
            // Near ties go to this CTA's region of the list: from the live-token
            // index of its first unit, as many entries as its units hold tokens.
            misc[8] = (int)(target * N + (lu0 % nblk) * KM_TOK);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    const int nunits = misc[4];
    const KpWalk start{misc[5], misc[6]};

    if (warp == 0) {
        // ------------------------------------------------------------ producer (lane 0)
        if (lane == 0 && nunits > 0) {
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_chi);
            prefetch_tmap(&tm_clo);
            KpWalk w = start;
            int i = 0, hs = -1, cur = -1;
            for (; i < nunits; ++i, w.next(state, BH, nblk)) {
                if (w.bh != cur) {  // the head's centroids, once the MMAs of the last head are done
                    if (hs >= 0 && !mbar_wait(b_cempty, hs & 1, ctl, abort_flag)) break;
                    ++hs;
                    cur = w.bh;
                    mbar_expect_tx_arrive(b_cfull, 2 * L.c_bytes);
#pragma unroll
                    for (int kc = 0; kc < D / 64; ++kc) {
                        tma_load_3d(base + L.off_chi + kc * (Cp * 128), &tm_chi, b_cfull, 64 * kc, 0, w.bh);
                        tma_load_3d(base + L.off_clo + kc * (Cp * 128), &tm_clo, b_cfull, 64 * kc, 0, w.bh);
                    }
                }
                const int st = i % S;
                if (i >= S && !mbar_wait(b_vempty(st), ((i / S) - 1) & 1, ctl, abort_flag)) break;
                mbar_expect_tx_arrive(b_vfull(st), L.v_bytes);
#pragma unroll
                for (int kc = 0; kc < D / 64; ++kc)
                    tma_load_3d(base + L.off_v + st * L.v_bytes + kc * (KM_TOK * 128), &tm_v, b_vfull(st),
                                64 * kc, w.tile * KM_TOK, w.bh);
            }
            // the copies still in flight (the earlier ones were consumed) land
            // before shared memory is released
            for (int j = i - S < 0 ? 0 : i - S; j < i; ++j) drain_wait(b_vfull(j % S), (j / S) & 1, ctl);
            if (hs >= 0) drain_wait(b_cfull, hs & 1, ctl);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (lane 0)
        if (lane == 0 && nunits > 0) {
            const uint32_t idesc = idesc_bf16_f32(Cp);
            KpWalk w = start;
            int hs = -1, cur = -1;
            for (int i = 0; i < nunits; ++i, w.next(state, BH, nblk)) {
                if (w.bh != cur) {
                    if (hs >= 0) mma_commit(b_cempty);  // the last head's MMAs: its centroids are free
                    ++hs;
                    cur = w.bh;
                    if (!mbar_wait(b_cfull, hs & 1, ctl, abort_flag)) break;
                }
                const int st = i % S, b = i % NACC;
                if (!mbar_wait(b_vfull(st), (i / S) & 1, ctl, abort_flag)) break;
                if (i >= NACC && !mbar_wait(b_accempty(b), ((i / NACC) - 1) & 1, ctl, abort_flag)) break;
                tc_fence_after();
                const uint32_t sA = base + L.off_v + st * L.v_bytes, acc = tmem + b * Cp;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    mma_bf16(acc, smem_desc(sA + (kk >> 2) * (KM_TOK * 128) + off, 128),
                             smem_desc(base + L.off_chi + (kk >> 2) * (Cp * 128) + off, 128), idesc, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    mma_bf16(acc, smem_desc(sA + (kk >> 2) * (KM_TOK * 128) + off, 128),
                             smem_desc(base + L.off_clo + (kk >> 2) * (Cp * 128) + off, 128), idesc, 1u);
                }
                mma_commit(b_accfull(b));
                mma_commit(b_vempty(st));
            }
            mma_commit(b_mmadone);  // every MMA issued has finished before TMEM is released
            drain_wait(b_mmadone, 0, ctl);
        }
    } else if (warp < 2 + ASG) {
        // ------------------------------------------------------------ assignment (thread per token)
        // Group g takes tiles i = g, g + G, ...  TMEM lane quadrant q = warp % 4
        // holds tile rows 32q..32q+31.
        const int g = (warp - 2) >> 2;
        const int qd = warp & 3;
        const int r = qd * 32 + lane;
        const int bar_id = 1 + g;
        float* cn_s = reinterpret_cast<float*>(smem + L.off_cn) + g * 64;
        uint32_t* cmax_s = reinterpret_cast<uint32_t*>(smem + L.off_cn) + G * 64 + g;
        uint8_t* ord_s = smem + L.off_ord;
        uint8_t* slab_s = smem + L.off_slab;
        int* seg_s = reinterpret_cast<int*>(smem + L.off_seg);
        uint8_t* ord2_s = smem + L.off_ord2;
        uint8_t* slab2_s = smem + L.off_slab2;
        int* seg2_s = reinterpret_cast<int*>(smem + L.off_seg2);
        const int tie_base = misc[8];
        KpWalk w = start;
        for (int q = 0; q < g; ++q) w.next(state, BH, nblk);
        int cur = -1, changed = 0;
        float cmax_r = 0.0f;
        auto flush_changed = [&]() {
            const int t = __reduce_add_sync(0xffffffffu, changed);
            if (lane == 0 && t) atomicAdd(&state[cur].chg[it & 1], t);
            changed = 0;
        };
        // the previous pass's label and |v|^2 of this thread's token, fetched
        // one group tile ahead so the loads overlap the work on the current one
        int32_t nxt_old = -1;
        float nxt_vn2 = 0.0f;
        auto fetch = [&](const KpWalk& u) {
            const int n = u.tile * KM_TOK + r;
            nxt_old = -1;
            nxt_vn2 = 0.0f;
            if (it > 0 && n < N) {
                nxt_old = labels[(size_t)u.bh * N + n];
                nxt_vn2 = vnorm2[(size_t)u.bh * N + n];
            }
        };
        if (g < nunits) fetch(w);
        for (int i = g; i < nunits; i += G) {
            const int bh = w.bh, tile = w.tile;
            if (bh != cur) {  // |c_k|^2 of the new head (pad clusters +inf, never chosen), max_k |c_k|^2
                if (cur >= 0) flush_changed();
                cur = bh;
                named_barrier_sync(bar_id, 128);  // every warp of the group is past the last head's tile
                if (qd == 0) {
                    uint32_t mb = 0;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int k = 2 * lane + e;
                        const float x = k < C ? cnorm[(size_t)bh * Cp + k] : INFINITY;
                        cn_s[k] = x;
                        if (k < C) mb = max(mb, __float_as_uint(x));  // x >= 0: bit order is value order
                    }
                    mb = __reduce_max_sync(0xffffffffu, mb);
                    if (lane == 0) *cmax_s = mb;
                }
                named_barrier_sync(bar_id, 128);
                cmax_r = sqrtf(__uint_as_float(*cmax_s));
            }
            const int32_t old_label = nxt_old;
            float vn2 = nxt_vn2;
#pragma unroll
            for (int q = 0; q < G; ++q) w.next(state, BH, nblk);  // this group's next tile
            if (i + G < nunits) fetch(w);
            const int st = i % S, b = i % NACC;
            // this tile's label counts: all valid tokens, the add list, the subtract list
            int* cnt = cnt_s + (g * 2 + ((i / G) & 1)) * 3 * 64;
            int* cnt_add = cnt + 64;
            int* cnt_sub = cnt + 128;
            const int n = tile * KM_TOK + r;
            const bool valid = n < N;
            // the accumulator of tile i (its MMA also means V tile i has landed)
            const bool okj = warp_wait(b_accfull(b), (i / NACC) & 1, ctl, abort_flag);
            int label = 0, rank = 0, rank_sub = 0;
            bool in_add = false, in_sub = false;
            if (okj) {
                tc_fence_after();
                const uint32_t lane_tmem = tmem + b * Cp + ((uint32_t)(qd * 32) << 16);
                float dk[64];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (16 * q < Cp) {
                        tmem_ld16(lane_tmem + 16 * q, dk + 16 * q);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) dk[16 * q + e] = 0.0f;  // pad clusters: |c|^2 = +inf decides
                    }
                }
                if (it == 0) {  // |v|^2 once per prep, from the V tile (resident until this warp releases it)
                    const uint8_t* arow = smem + L.off_v + st * L.v_bytes + r * 128;
                    vn2 = 0.0f;
#pragma unroll
                    for (int kc = 0; kc < D / 64; ++kc)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            const uint4 raw = *reinterpret_cast<const uint4*>(arow + kc * (KM_TOK * 128) +
                                                                              ((ch ^ (r & 7)) << 4));
                            const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                            for (int e = 0; e < 8; ++e) vn2 = fmaf(bf2f(hv[e]), bf2f(hv[e]), vn2);
                        }
                    if (valid) vnorm2[(size_t)bh * N + n] = vn2;
                }
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_accempty(b));  // the accumulator is free for tile i + NACC
                // best and runner-up of d_k = |c_k|^2 - 2 v.c_k, four chains (k % 4)
                float b4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
                float s4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
                int k4[4] = {0, 0, 0, 0};
#pragma unroll
                for (int q4 = 0; q4 < 16; ++q4) {
                    const float4 cn = reinterpret_cast<const float4*>(cn_s)[q4];
                    const float cv[4] = {cn.x, cn.y, cn.z, cn.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float d = fmaf(-2.0f, dk[4 * q4 + e], cv[e]);
                        dk[4 * q4 + e] = d;
                        const bool lt = d < b4[e];
                        s4[e] = fminf(s4[e], fmaxf(b4[e], d));
                        b4[e] = fminf(b4[e], d);
                        k4[e] = lt ? 4 * q4 + e : k4[e];
                    }
                }
                float best = b4[0], second = s4[0];
                int bestk = k4[0];
#pragma unroll
                for (int e = 1; e < 4; ++e) {
                    second = fminf(fminf(second, s4[e]), fmaxf(best, b4[e]));
                    if (b4[e] < best || (b4[e] == best && k4[e] < bestk)) {
                        best = b4[e];
                        bestk = k4[e];
                    }
                }
                // Near ties within the error bound derived at km_assign.  The
                // radius takes an approximate square root (relative error near
                // 2^-22): the margin sits 2.6 times above the bound, and only
                // chooses which tokens km_refine decides again in fp64.
                const float rad = (vn2 > 0.0f ? vn2 * rsqrtf(vn2) : 0.0f) + cmax_r;
                const float margin = rad * rad * 0x1p-13f;
                const bool refine = valid && C > 1 && (second - best) <= margin;
                const uint32_t rmask = __ballot_sync(0xffffffffu, refine);
                if (rmask != 0) {
                    int first = 0;
                    if (lane == 0) first = atomicAdd(tie_s, __popc(rmask));
                    first = __shfl_sync(0xffffffffu, first, 0);
                    if (refine) {
                        KmTie* e = ties + tie_base + first + __popc(rmask & ((1u << lane) - 1));
                        const float lim = best + margin;
                        uint32_t m0 = 0, m1 = 0;  // candidates 0..31 and 32..63 (pads are +inf)
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            if (dk[jj] <= lim) m0 |= 1u << jj;
                            if (dk[32 + jj] <= lim) m1 |= 1u << jj;
                        }
                        e->mask[0] = m0;
                        e->mask[1] = m1;
                        *reinterpret_cast<int4*>(e) = make_int4(bh, n, old_label, bestk);
                    }
                }
                if (valid) {
                    label = bestk;
                    if (it == 0 || old_label != label) ++changed;
                    labels[(size_t)bh * N + n] = label;
                    // the token's place among its cluster's in this tile's lists
                    in_add = mode == 1 || (mode == 3 && old_label != label);
                    in_sub = mode == 3 && old_label != label;
                    if (in_add) rank = atomicAdd(&cnt_add[label], 1);
                    if (in_sub) rank_sub = atomicAdd(&cnt_sub[old_label], 1);
                    if (mode != 1) atomicAdd(&cnt[label], 1);  // mode 1: the add list is the histogram
                }
                if (mode == 2) {  // move the tokens that changed cluster, a row at a time over the warp
                    constexpr int NCH = D / 32;
                    const int c0 = NCH * lane;
                    const uint8_t* vtile = smem + L.off_v + st * L.v_bytes + (c0 >> 6) * (KM_TOK * 128) + (c0 & 7) * 2;
                    const int q16 = (c0 & 63) >> 3;
                    uint32_t cm = __ballot_sync(0xffffffffu, valid && label != old_label);
                    while (cm) {
                        const int src = __ffs(cm) - 1;
                        cm &= cm - 1;
                        const int ko = __shfl_sync(0xffffffffu, old_label, src);
                        const int kn = __shfl_sync(0xffffffffu, label, src);
                        const int row = qd * 32 + src;
                        const uint8_t* p2 = vtile + row * 128 + ((q16 ^ (row & 7)) << 4);
                        double* so = sums + ((size_t)bh * C + ko) * D + c0;
                        double* sn = sums + ((size_t)bh * C + kn) * D + c0;
#pragma unroll
                        for (int h = 0; h < NCH / 2; ++h) {
                            const uint32_t w2 = reinterpret_cast<const uint32_t*>(p2)[h];
                            const double x0 = bf16lo_scaled(w2) * kBf16Unscale;  // exact
                            const double x1 = bf16hi_scaled(w2) * kBf16Unscale;
                            atomicAdd(so + 2 * h, -x0);
                            atomicAdd(so + 2 * h + 1, -x1);
                            atomicAdd(sn + 2 * h, x0);
                            atomicAdd(sn + 2 * h + 1, x1);
                        }
                    }
                }
            }
            // one decision for the four warps: leave together or go on together
            if (!named_barrier_and(bar_id, 128, okj)) break;
            int* seg = seg_s + st * KP_SEG;
            int* seg2 = seg2_s + st * KP_SEG;
            if (qd == 0) {  // the tile's histogram, to global; cluster offsets for the grouping
                const int k0 = 2 * lane;
                // counts of clusters k0, k0 + 1 in one list, zeroed for this group's tile after next;
                // with `seg`, that list's exclusive scan over the clusters
                auto take = [&](int* cn, int* sg) {
                    const int h0 = cn[k0], h1 = cn[k0 + 1];
                    cn[k0] = 0;
                    cn[k0 + 1] = 0;
                    if (sg) {
                        int x = h0 + h1;
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const int y = __shfl_up_sync(0xffffffffu, x, o);
                            if (lane >= o) x += y;
                        }
                        sg[k0] = x - h0 - h1;
                        sg[k0 + 1] = x - h1;
                        if (lane == 31) sg[64] = x;
                    }
                    return make_int2(h0, h1);
                };
                const int2 h = mode == 1 ? take(cnt_add, seg) : take(cnt, nullptr);
                if (mode == 3) {
                    take(cnt_add, seg);
                    take(cnt_sub, seg2);
                }
                if (k0 < C) hist[((size_t)bh * C + k0) * nblk + tile] = h.x;
                if (k0 + 1 < C) hist[((size_t)bh * C + k0 + 1) * nblk + tile] = h.y;
            }
            if (accumulate) {
                named_barrier_sync(bar_id, 128);
                if (in_add) {
                    const int pos = st * KM_TOK + seg[label] + rank;
                    ord_s[pos] = (uint8_t)r;
                    slab_s[pos] = (uint8_t)label;
                }
                if (in_sub) {
                    const int pos = st * KM_TOK + seg2[old_label] + rank_sub;
                    ord2_s[pos] = (uint8_t)r;
                    slab2_s[pos] = (uint8_t)old_label;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(b_lfull(st));  // the tile's grouping, for the update warps
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b_vempty(st));
        }
        if (cur >= 0) flush_changed();
    } else if (UPD && accumulate && nunits > 0) {
        // ------------------------------------------------------------ update, modes 1 and 3 (D/32 channels a lane)
        constexpr int NCH = D / 32;
        const int u = warp - 2 - ASG;           // clusters CPW u .. CPW u + CPW - 1
        const int c0 = NCH * lane;              // channels c0 .. c0 + NCH - 1
        const int kc = c0 >> 6, q16 = (c0 & 63) >> 3, wo = (c0 & 7) * 2;  // chunk, 16-byte piece, byte
        auto flush = [&](int bh) {  // this warp's sums of head bh to the global sums, then zero
#pragma unroll 1
            for (int k = CPW * u; k < CPW * u + CPW && k < C; ++k) {
#pragma unroll
                for (int e = 0; e < NCH; ++e) {
                    double* sp = sums_s + k * D + c0 + e;
                    if (*sp != 0.0) atomicAdd(&sums[((size_t)bh * C + k) * D + c0 + e], *sp * kBf16Unscale);
                    *sp = 0.0;
                }
            }
        };
        KpWalk w = start;
        int cur = -1;
        bool ok = true;
        for (int i = 0; i < nunits; ++i, w.next(state, BH, nblk)) {
            if (w.bh != cur) {
                if (cur >= 0) flush(cur);
                cur = w.bh;
            }
            const int st = i % S;
            // the update trails the assignment by a tile: wait without polling hard
            if (!(ok = warp_wait_idle(b_lfull(st), (i / S) & 1, ctl, abort_flag, 100))) break;
            const uint8_t* vt = smem + L.off_v + st * L.v_bytes + kc * (KM_TOK * 128) + wo;
            // One grouped list of the tile: the warp's clusters hold its
            // positions [P0, P1); each run is added to (or subtracted from)
            // the CTA's sums.
            auto walk = [&](uint32_t off_ord, uint32_t off_slab, uint32_t off_seg, bool subtract) {
                const uint8_t* ord = smem + off_ord + st * KM_TOK;
                const uint8_t* slab = smem + off_slab + st * KM_TOK;
                const int* segp = reinterpret_cast<const int*>(smem + off_seg) + st * KP_SEG + CPW * u;
                const int P0 = segp[0], P1 = segp[CPW];
                double run[NCH];
#pragma unroll
                for (int e = 0; e < NCH; ++e) run[e] = 0.0;
                int rk = P0 < P1 ? slab[P0] : 0;  // cluster of the run being added
                auto flush_run = [&]() {
                    double* sp = sums_s + rk * D + c0;
#pragma unroll
                    for (int e = 0; e < NCH; ++e) {
                        sp[e] = subtract ? sp[e] - run[e] : sp[e] + run[e];
                        run[e] = 0.0;
                    }
                };
#pragma unroll 1
                for (int p = P0; p < P1; p += 4) {
                    // four positions' rows and clusters first, so their loads overlap
                    int j[4], kk[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int pp = min(p + t, P1 - 1);
                        j[t] = ord[pp];
                        kk[t] = p + t < P1 ? (int)slab[pp] : -1;
                    }
                    uint32_t x[4][NCH / 2];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint8_t* src = vt + j[t] * 128 + ((q16 ^ (j[t] & 7)) << 4);  // row j, 128-byte swizzle
                        if constexpr (NCH == 4) {
                            const uint2 y = *reinterpret_cast<const uint2*>(src);
                            x[t][0] = y.x;
                            x[t][1] = y.y;
                        } else {
                            x[t][0] = *reinterpret_cast<const uint32_t*>(src);
                        }
                    }
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        if (kk[t] < 0) break;
                        if (kk[t] != rk) {  // a new cluster's run starts (uniform over the warp)
                            flush_run();
                            rk = kk[t];
                        }
#pragma unroll
                        for (int h = 0; h < NCH / 2; ++h) {
                            run[2 * h] += bf16lo_scaled(x[t][h]);
                            run[2 * h + 1] += bf16hi_scaled(x[t][h]);
                        }
                    }
                }
                if (P0 < P1) flush_run();
            };
            walk(L.off_ord, L.off_slab, L.off_seg, false);
            if (mode == 3) walk(L.off_ord2, L.off_slab2, L.off_seg2, true);
            __syncwarp();
            if (lane == 0) mbar_arrive(b_vempty(st));
        }
        if (ok && cur >= 0) flush(cur);
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {  // this CTA's near-tie region for km_refine
        tie_regions[2 * blockIdx.x] = misc[8];
        tie_regions[2 * blockIdx.x + 1] = *tie_s;
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

// Decision of the near ties km_assign or km_pass listed, by the Lloyd step's
// own distance (the fp64 sum over channels of (v - c)^2, argmin with equal
// distances keeping the lowest cluster).  When the decision differs from the
// tensor-core label, the label, the tile's cluster counts, the head's change
// count and (when the sums are kept) the sums are corrected.  The list is
// either one run counted in tie_count[it % 2] (km_assign) or, with nreg > 0,
// km_pass's per-CTA regions: (start, count) pairs in tie_regions.
//
// Most ties are settled first in fp32 from the bf16 hi/lo centroids.
// c32 = hi + lo lies within 2^-17.9 |c_i| of the fp64 centroid in every
// channel (two bf16 roundings, and the fp32 sum), so D(c32) is within
// 2^-16.9 sqrt(D) |c| + 2^-35.8 |c|^2 of D(c); the fp32 evaluation
// (differences, then d/8 fused multiply-adds a lane and a three-level
// butterfly: at most 20 roundings on any term) adds at most 2^-19.6 D.  With
// each term doubled, E = 2^-16 sqrt(D32) |c| + 2^-35 |c|^2 + 2^-18 D32 bounds
// |D32 - D|.  A candidate whose D32 + E is below every other candidate's
// D32 - E is the exact argmin; otherwise all candidates are compared in fp64
// from the fp64 centroids, in ascending cluster order with a strict
// comparison.
template <int D>
__global__ void __launch_bounds__(256) km_refine(const KmTie* __restrict__ ties, int* __restrict__ tie_count,
                                                 const int* __restrict__ tie_regions, int nreg,
                                                 const __nv_bfloat16* __restrict__ c_hi,
                                                 const __nv_bfloat16* __restrict__ c_lo,
                                                 const float* __restrict__ cnorm,
                                                 const __nv_bfloat16* __restrict__ V,
                                                 const double* __restrict__ cent64, int32_t* __restrict__ labels,
                                                 int32_t* __restrict__ hist, double* __restrict__ sums,
                                                 KmState* __restrict__ state, int N, int C, int Cp, int it,
                                                 int accumulate, const int* __restrict__ status) {
    __shared__ int pre_s[KP_MAX_GRID + 1];  // entries before each region
    __shared__ int start_s[KP_MAX_GRID];
    if (ctl_failed(status)) return;
    int count;
    if (nreg > 0) {
        if (threadIdx.x < 32) {  // exclusive prefix of the region counts, 32 at a time
            int carry = 0;
            for (int r0 = 0; r0 < nreg; r0 += 32) {
                const int r = r0 + threadIdx.x;
                const int c = r < nreg ? tie_regions[2 * r + 1] : 0;
                if (r < nreg) start_s[r] = tie_regions[2 * r];
                int x = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, x, o);
                    if ((int)threadIdx.x >= o) x += y;
                }
                if (r < nreg) pre_s[r] = carry + x - c;
                carry += __shfl_sync(0xffffffffu, x, 31);
            }
            if (threadIdx.x == 0) pre_s[nreg] = carry;
        }
        __syncthreads();
        count = pre_s[nreg];
    } else {
        count = tie_count[it & 1];
        if (blockIdx.x == 0 && threadIdx.x == 0) tie_count[(it + 1) & 1] = 0;  // the next pass's list starts empty
    }
    // Four ties a warp, eight lanes a tie (D/8 channels a lane): four ties'
    // loads in flight at once.  Loops over candidate slots run the same count
    // on every lane (the warp's largest candidate count), so every shuffle
    // is reached by all 32 lanes.
    constexpr int TL = 8, TPW = 32 / TL, CPT = D / TL;
    const int lane = threadIdx.x & 31, sub = lane / TL, sl = lane % TL;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nblk = (N + KM_TOK - 1) / KM_TOK;
    const int words = (Cp + 31) >> 5;
    for (int base = gw * TPW; base < count; base += nwarps * TPW) {
        const int e0 = base + sub;
        const bool act = e0 < count;
        int e = e0;
        if (act && nreg > 0) {  // the region holding entry e0: the last r with pre_s[r] <= e0 (never an empty one)
            int lo = 0, hi = nreg - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (pre_s[mid] <= e0) lo = mid; else hi = mid - 1;
            }
            e = start_s[lo] + e0 - pre_s[lo];
        }
        const int4 hd = act ? *reinterpret_cast<const int4*>(ties + e) : make_int4(0, 0, -1, -1);  // bh, n, old, prov
        const int bh = hd.x, n = hd.y;
        float vx[CPT];
        {
            const uint4* vp = reinterpret_cast<const uint4*>(V + ((size_t)bh * N + n) * D + sl * CPT);
#pragma unroll
            for (int q = 0; q < CPT / 8; ++q) {
                const uint4 x = act ? __ldg(vp + q) : make_uint4(0, 0, 0, 0);
                const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    vx[8 * q + 2 * h] = __uint_as_float(w4[h] << 16);
                    vx[8 * q + 2 * h + 1] = __uint_as_float(w4[h] & 0xFFFF0000u);
                }
            }
        }
        int nc = 0;
        for (int w = 0; act && w < words; ++w) nc += __popc(ties[e].mask[w]);
        const int ncmax = __reduce_max_sync(0xffffffffu, nc);
        // fp32 bounds of every candidate's distance (uniform over the tie's lanes)
        float umin = INFINITY, lmin1 = INFINITY, lmin2 = INFINITY;
        int ku = -1, kl1 = -1;
        int cw = 0;
        uint32_t bits = act ? ties[e].mask[0] : 0u;
        for (int j = 0; j < ncmax; ++j) {
            while (bits == 0 && act && cw + 1 < words) bits = ties[e].mask[++cw];
            const bool has = bits != 0;
            const int k = has ? 32 * cw + __ffs(bits) - 1 : 0;
            bits &= bits - 1;
            float part = 0.0f;
            if (has) {
                const size_t row = ((size_t)bh * Cp + k) * D + sl * CPT;
#pragma unroll
                for (int q = 0; q < CPT / 8; ++q) {
                    const uint4 h4 = __ldg(reinterpret_cast<const uint4*>(c_hi + row) + q);
                    const uint4 l4 = __ldg(reinterpret_cast<const uint4*>(c_lo + row) + q);
                    const uint32_t hw[4] = {h4.x, h4.y, h4.z, h4.w}, lw[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float c0 = __fadd_rn(__uint_as_float(hw[h] << 16), __uint_as_float(lw[h] << 16));
                        const float c1 = __fadd_rn(__uint_as_float(hw[h] & 0xFFFF0000u),
                                                   __uint_as_float(lw[h] & 0xFFFF0000u));
                        const float d0 = __fsub_rn(vx[8 * q + 2 * h], c0);
                        const float d1 = __fsub_rn(vx[8 * q + 2 * h + 1], c1);
                        part = __fmaf_rn(d0, d0, part);
                        part = __fmaf_rn(d1, d1, part);
                    }
                }
            }
#pragma unroll
            for (int o = TL / 2; o > 0; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
            if (has) {
                const float c2 = cnorm[(size_t)bh * Cp + k];
                const float err = 0x1p-16f * sqrtf(part * c2) + 0x1p-35f * c2 + 0x1p-18f * part;
                const float up = part + err, lo = part - err;
                if (up < umin) {
                    umin = up;
                    ku = k;
                }
                if (lo < lmin1) {
                    lmin2 = lmin1;
                    lmin1 = lo;
                    kl1 = k;
                } else if (lo < lmin2) {
                    lmin2 = lo;
                }
            }
        }
        // the fp32 winner is certain when its upper bound is below every other lower bound
        const bool sure = ku >= 0 && umin < (kl1 == ku ? lmin2 : lmin1);
        int kbest = sure ? ku : hd.w;
        const bool need = act && !sure;
        if (__any_sync(0xffffffffu, need)) {
            // fp64 decision: candidates in ascending order, strict comparison
            // (equal distances keep the lowest cluster, as the Lloyd argmin)
            double dbest = INFINITY;
            cw = 0;
            bits = need ? ties[e].mask[0] : 0u;
            for (int j = 0; j < ncmax; ++j) {
                while (bits == 0 && need && cw + 1 < words) bits = ties[e].mask[++cw];
                const bool has = bits != 0;
                const int k = has ? 32 * cw + __ffs(bits) - 1 : 0;
                bits &= bits - 1;
                double part = 0.0;
                if (has) {
                    const double2* cp =
                        reinterpret_cast<const double2*>(cent64 + ((size_t)bh * C + k) * D + sl * CPT);
#pragma unroll
                    for (int i = 0; i < CPT / 2; ++i) {
                        const double2 c2 = __ldg(cp + i);
                        const double d0 = __dsub_rn((double)vx[2 * i], c2.x);
                        const double d1 = __dsub_rn((double)vx[2 * i + 1], c2.y);
                        part = __dadd_rn(part, __dmul_rn(d0, d0));
                        part = __dadd_rn(part, __dmul_rn(d1, d1));
                    }
                }
#pragma unroll
                for (int o = TL / 2; o > 0; o >>= 1) part = __dadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
                if (has && part < dbest) {
                    dbest = part;
                    kbest = k;
                }
            }
        }
        if (act && kbest != hd.w) {  // uniform over the tie's lanes
            if (accumulate) {  // the token's channels move from the tensor-core cluster's sums to the new one's
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    atomicAdd(&sums[((size_t)bh * C + hd.w) * D + sl * CPT + i], -(double)vx[i]);
                    atomicAdd(&sums[((size_t)bh * C + kbest) * D + sl * CPT + i], (double)vx[i]);
                }
            }
            if (sl == 0) {
                labels[(size_t)bh * N + n] = kbest;
                const int tile = n / KM_TOK;
                atomicSub(&hist[((size_t)bh * C + hd.w) * nblk + tile], 1);
                atomicAdd(&hist[((size_t)bh * C + kbest) * nblk + tile], 1);
                const int dchg = (kbest != hd.z) - (hd.w != hd.z);
                if (dchg != 0) atomicAdd(&state[bh].chg[it & 1], dchg);
            }
        }
    }
}

// Exclusive scan of hist[bh] in (cluster, block) order -> offs; cluster ranges.
// The histogram goes through shared memory in chunks of KM_SCAN_CHUNK entries:
// loaded and stored coalesced, scanned as 1024 contiguous runs of 16 plus a
// block scan of the run totals, with a carry between chunks.
constexpr int KM_SCAN_CHUNK = 16 * 1024;

__global__ void __launch_bounds__(1024) km_scan(const int32_t* __restrict__ hist, int32_t* __restrict__ offs,
                                                int32_t* __restrict__ cstart, int32_t* __restrict__ ccount,
                                                KmState* __restrict__ state, int N, int C, int nblk, int it,
                                                int decide, const int* __restrict__ status) {
    extern __shared__ int h_s[];  // [KM_SCAN_CHUNK]
    __shared__ int s_part[1024];
    __shared__ int s_skip;
    if (ctl_failed(status)) return;
    const int bh = blockIdx.x, tid = threadIdx.x;
    if (tid == 0) {
        int skip = 0;
        if (decide) {  // per pass: a head whose labels repeat the previous pass is final
            skip = state[bh].done;
            if (!skip && it > 0 && state[bh].chg[it & 1] == 0) {
                state[bh].done = 1;
                skip = 1;
            }
            if (!skip) state[bh].chg[it & 1] = 0;  // for pass it + 2
        }
        s_skip = skip;
    }
    __syncthreads();
    if (s_skip) return;
    const int64_t L = (int64_t)C * nblk;
    const int32_t* hh = hist + (size_t)bh * L;
    int32_t* oo = offs + (size_t)bh * L;
    int carry = 0;
    for (int64_t c0 = 0; c0 < L; c0 += KM_SCAN_CHUNK) {
        const int n = (int)(L - c0 < KM_SCAN_CHUNK ? L - c0 : KM_SCAN_CHUNK);
        for (int i = tid; i < n; i += 1024) h_s[i] = hh[c0 + i];
        __syncthreads();
        const int a = min(n, 16 * tid), b = min(n, a + 16);
        int sum = 0;
        for (int i = a; i < b; ++i) sum += h_s[i];
        s_part[tid] = sum;
        __syncthreads();
        for (int d = 1; d < 1024; d <<= 1) {
            const int v = tid >= d ? s_part[tid - d] : 0;
            __syncthreads();
            s_part[tid] += v;
            __syncthreads();
        }
        int run = carry + s_part[tid] - sum;  // exclusive prefix of this run
        for (int i = a; i < b; ++i) {
            const int x = h_s[i];
            h_s[i] = run;
            run += x;
        }
        const int total = s_part[1023];
        __syncthreads();
        for (int i = tid; i < n; i += 1024) oo[c0 + i] = h_s[i];
        carry += total;
        __syncthreads();
    }
    __syncthreads();
    for (int k = tid; k < C; k += 1024) {
        const int st = oo[(int64_t)k * nblk];
        const int en = k + 1 < C ? oo[(int64_t)(k + 1) * nblk] : N;
        cstart[(size_t)bh * C + k] = st;
        ccount[(size_t)bh * C + k] = en - st;
    }
}

// perm[position] = token, stable within a cluster: a token's position is its
// cluster's offset for this tile plus the number of earlier tokens of the
// tile with the same cluster (within its warp by __match_any_sync, plus the
// counts of the earlier warps).
__global__ void __launch_bounds__(KM_TOK) km_scatter(const int32_t* __restrict__ labels,
                                                     const int32_t* __restrict__ offs, int32_t* __restrict__ perm,
                                                     const KmState* __restrict__ state, int N, int C,
                                                     int skip_done, const int* __restrict__ status) {
    __shared__ int cnt_s[KM_TOK / 32][256];
    const int bh = blockIdx.y, blk = blockIdx.x, nblk = gridDim.x, r = threadIdx.x;
    if (ctl_failed(status) || (skip_done && state[bh].done)) return;
    const int warp = r >> 5, lane = r & 31;
    for (int i = r; i < (KM_TOK / 32) * 256; i += KM_TOK) (&cnt_s[0][0])[i] = 0;
    const int j = blk * KM_TOK + r;
    const int L = j < N ? labels[(size_t)bh * N + j] : -1;
    const uint32_t same = __match_any_sync(0xffffffffu, L);
    __syncthreads();
    if (L >= 0 && lane == __ffs(same) - 1) cnt_s[warp][L] = __popc(same);
    __syncthreads();
    if (L < 0) return;
    int rank = __popc(same & ((1u << lane) - 1));
    for (int w = 0; w < warp; ++w) rank += cnt_s[w][L];
    perm[(size_t)bh * N + offs[((size_t)bh * C + L) * nblk + blk] + rank] = j;
}

// fp64 member sums for the Lloyd update.  The stable order lists the members
// of cluster 0, then cluster 1, ...; one CTA takes a fixed slice of KM_UPD_ROWS
// positions of it (so large clusters spread over many CTAs) and walks the
// cluster segments inside the slice: a row is read as D/8 16-byte pieces (8
// channels a thread), the row groups are added in shared memory, and each
// segment adds its sum to `sums` with one fp64 atomic per channel.
constexpr int KM_UPD_ROWS = 256;

template <int D>
__global__ void __launch_bounds__(128) km_update(const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ perm,
                                                 const int32_t* __restrict__ cstart, double* __restrict__ sums,
                                                 const KmState* __restrict__ state, int N, int C,
                                                 const int* __restrict__ status) {
    constexpr int TPR = D / 8;    // threads per row
    constexpr int R = 128 / TPR;  // rows per pass
    __shared__ double red[R][D];
    __shared__ int pp_s[KM_UPD_ROWS];
    __shared__ int seg_s;
    const int bh = blockIdx.y;
    if (ctl_failed(status) || state[bh].done) return;
    const int r0 = blockIdx.x * KM_UPD_ROWS, r1 = min(N, r0 + KM_UPD_ROWS);
    const int tid = threadIdx.x, cg = tid % TPR, rr = tid / TPR;
    const int32_t* cs = cstart + (size_t)bh * C;
    if (tid == 0) {  // the cluster holding position r0: the last k with cstart[k] <= r0
        int lo = 0, hi = C - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cs[mid] <= r0) lo = mid; else hi = mid - 1;
        }
        seg_s = lo;
    }
    __syncthreads();
    const uint4* vb = reinterpret_cast<const uint4*>(V + (size_t)bh * N * D) + cg;
    for (int i = tid; i < r1 - r0; i += 128) pp_s[i] = perm[(size_t)bh * N + r0 + i];
    __syncthreads();
    const int* pp = pp_s - r0;  // indexed by position
    for (int k = seg_s; k < C; ++k) {
        const int a = max(r0, cs[k]);
        const int b = min(r1, k + 1 < C ? cs[k + 1] : N);
        if (a >= r1) break;
        if (b <= a) continue;  // empty cluster (uniform over the CTA)
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
        auto add = [&](const uint4& x) {
            const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __dadd_rn(acc[e], (double)bf2f(h[e]));
        };
        int i = a + rr;
        for (; i + 7 * R < b; i += 8 * R) {
            uint4 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = __ldg(vb + (size_t)pp[i + u * R] * TPR);
#pragma unroll
            for (int u = 0; u < 8; ++u) add(x[u]);
        }
        for (; i < b; i += R) add(__ldg(vb + (size_t)pp[i] * TPR));
#pragma unroll
        for (int e = 0; e < 8; ++e) red[rr][cg * 8 + e] = acc[e];
        __syncthreads();
        for (int c = tid; c < D; c += 128) {
            double t = 0.0;
#pragma unroll
            for (int q = 0; q < R; ++q) t = __dadd_rn(t, red[q][c]);
            atomicAdd(&sums[((size_t)bh * C + k) * D + c], t);
        }
        __syncthreads();
    }
}

// Lloyd update: c_k = sum / count in fp64 (empty clusters keep c_k), as bf16
// hi/lo, fp32 |c_k|^2 and fp64 for km_refine; the sums are zeroed for the next
// pass, or kept (keep_sums) when the next pass moves only the tokens that
// change cluster.  The counts come from km_scan (ccount) or, after km_pass, from the
// tile histograms; then the pass's change count also decides here whether
// the head is final (its labels repeat the previous pass, so the centroids
// would not move).
__global__ void km_finalize(__nv_bfloat16* __restrict__ c_hi, __nv_bfloat16* __restrict__ c_lo,
                            float* __restrict__ cnorm, double* __restrict__ cent64, double* __restrict__ sums,
                            const int32_t* __restrict__ ccount, const int32_t* __restrict__ hist,
                            KmState* __restrict__ state, int C, int Cp, int D, int nblk, int it, int from_hist,
                            int keep_sums, const int* __restrict__ status) {
    __shared__ float red[4];
    __shared__ int red_i[4];
    const int k = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
    if (ctl_failed(status) || state[bh].done) return;
    int cnt;
    if (from_hist) {
        // every CTA of the head reads the same count (no one writes it during this kernel)
        if (it >= 1 && state[bh].chg[it & 1] == 0) {
            if (k == 0 && c == 0) state[bh].done = 1;
            return;
        }
        if (k == 0 && c == 0) state[bh].chg[(it + 1) & 1] = 0;  // read last by the previous pass's finalize
        int part = 0;
        for (int t = c; t < nblk; t += D) part += hist[((size_t)bh * C + k) * nblk + t];
        part = __reduce_add_sync(0xffffffffu, part);
        if ((c & 31) == 0) red_i[c >> 5] = part;
        __syncthreads();
        cnt = 0;
        for (int w = 0; w < (D >> 5); ++w) cnt += red_i[w];
    } else {
        cnt = ccount[(size_t)bh * C + k];
    }
    if (cnt == 0) return;  // an empty cluster keeps its centroid (sums are still 0)
    double* sp = &sums[((size_t)bh * C + k) * D + c];
    const double mean = __ddiv_rn(*sp, (double)cnt);  // the fp64 member mean
    if (!keep_sums) *sp = 0.0;
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
// One CTA per (block of BK regrouped tokens, head), 256 threads.  The block's
// gathered K rows, then its V rows, are copied once, 16 bytes a piece with
// every piece of a thread in flight, into one shared buffer; every pass below
// works from there.  K: amax over the block, inv = 448/amax,
// code = E4M3(k * inv), k_scale = amax/448.  V: block mean (fp64 sum / valid,
// rounded to fp32; zero when smooth == 0), residual channel amax folded into
// vamax with an integer max on the fp32 bits (all >= 0).
constexpr int PREP_THREADS = 256;

// A regrouped position's token, forced into [0, N): a permutation passed in by
// the caller (the reuse mode) can then never index outside the head.
__device__ __forceinline__ int clamp_tok(int32_t t, int N) { return (uint32_t)t < (uint32_t)N ? t : 0; }

// One buffer of a block's rows: first its K rows, then its V rows, so that
// about six CTAs share an SM and some are always loading.
template <int D, int BK>
constexpr int kv_block_smem() {
    return BK * D * 2;
}

template <int D, int BK>
__global__ void __launch_bounds__(PREP_THREADS) prep_kv_block(const __nv_bfloat16* __restrict__ K,
                                                              const __nv_bfloat16* __restrict__ V,
                                                              const int32_t* __restrict__ perm, int smooth,
                                                              uint8_t* __restrict__ k_fp8, float* __restrict__ k_scale,
                                                              float* __restrict__ v_mean, uint32_t* __restrict__ vamax,
                                                              int N, int T, const int* __restrict__ status) {
    constexpr int NT = PREP_THREADS;
    constexpr int RG = NT / D;  // row groups of the per-channel passes
    constexpr int CH = D / 8;   // 16-byte pieces per row
    extern __shared__ uint4 kv_s[];  // the block's K rows [BK][CH], later its V rows
    __shared__ int tok_s[BK];
    __shared__ uint32_t red_s[NT / 32];
    __shared__ double vsum_s[RG][D];
    __shared__ float vmax_s[RG][D];
    if (ctl_failed(status)) return;  // perm is undefined
    const int b = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int valid = min(BK, N - b * BK);
    for (int r = tid; r < BK; r += NT) tok_s[r] = r < valid ? clamp_tok(perm[(size_t)bh * N + b * BK + r], N) : 0;
    __syncthreads();
    uint4* ks = kv_s;
    uint4* vs = kv_s;
    const uint4* kg = reinterpret_cast<const uint4*>(K + (size_t)bh * N * D);
    const uint4* vg = reinterpret_cast<const uint4*>(V + (size_t)bh * N * D);
#pragma unroll
    for (int u = 0; u < BK * CH / NT; ++u) {
        const int i = tid + u * NT;
        const int r = i / CH;
        if (r < valid) cp_async16(ks + i, kg + (size_t)tok_s[r] * CH + i % CH);
    }
    cp_async_wait_all();
    uint32_t kmax_bits = 0;  // |k| >= 0: the fp32 bit order is the value order
#pragma unroll
    for (int u = 0; u < BK * CH / NT; ++u) {  // the thread's own pieces
        const int i = tid + u * NT;
        if (i / CH < valid) {
            const uint4 kx = ks[i];
            const uint32_t w[4] = {kx.x, kx.y, kx.z, kx.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)  // bf16 -> fp32 bits of |k|: the high half, sign cleared
                kmax_bits = max(kmax_bits, max((w[e] << 16) & 0x7FFFFFFFu, w[e] & 0x7FFF0000u));
        }
    }
    kmax_bits = __reduce_max_sync(0xffffffffu, kmax_bits);
    if ((tid & 31) == 0) red_s[tid >> 5] = kmax_bits;
    __syncthreads();
    uint32_t am = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) am = max(am, red_s[w]);
    const float amax = __uint_as_float(am);
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
    if (tid == 0) k_scale[(size_t)bh * T + b] = __fdiv_rn(amax, 448.0f);

    const __nv_bfloat16* ksh = reinterpret_cast<const __nv_bfloat16*>(ks);
    const __nv_bfloat16* vsh = reinterpret_cast<const __nv_bfloat16*>(vs);
    const int c = tid % D, rg = tid / D;
    // K codes, four channels a thread (one 32-bit store); padding rows are 0
    uint32_t* kout = reinterpret_cast<uint32_t*>(k_fp8 + ((size_t)bh * T * BK + (size_t)b * BK) * D);
#pragma unroll 4
    for (int i = tid; i < BK * D / 4; i += NT) {
        const int r = i / (D / 4);
        uint32_t w = 0;
        if (r < valid) {
            const uint2 raw = reinterpret_cast<const uint2*>(ksh)[i];
            const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
            w = (uint32_t)e4m3x2(__fmul_rn(bf2f(h[0]), inv), __fmul_rn(bf2f(h[1]), inv)) |
                ((uint32_t)e4m3x2(__fmul_rn(bf2f(h[2]), inv), __fmul_rn(bf2f(h[3]), inv)) << 16);
        }
        kout[i] = w;
    }
    __syncthreads();  // every K row read: the buffer takes the V rows
#pragma unroll
    for (int u = 0; u < BK * CH / NT; ++u) {
        const int i = tid + u * NT;
        const int r = i / CH;
        if (r < valid) cp_async16(vs + i, vg + (size_t)tok_s[r] * CH + i % CH);
    }
    cp_async_wait_all();
    __syncthreads();
    // The channel's sum over the block in fp64, four partial sums of the
    // bf16 values placed as v * 2^-896 (exact, see bf16lo_scaled); scaled
    // back once below.  Exact additions make the order irrelevant.
    const uint16_t* vbits = reinterpret_cast<const uint16_t*>(vs);
    double vp[4] = {0.0, 0.0, 0.0, 0.0};
    int r = rg;
    for (; r + 3 * RG < valid; r += 4 * RG) {
#pragma unroll
        for (int e = 0; e < 4; ++e) vp[e] += bf16lo_scaled(vbits[(r + e * RG) * D + c]);
    }
    for (; r < valid; r += RG) vp[0] += bf16lo_scaled(vbits[r * D + c]);
    vsum_s[rg][c] = (vp[0] + vp[1]) + (vp[2] + vp[3]);
    __syncthreads();
    double tot = 0.0;
#pragma unroll
    for (int q = 0; q < RG; ++q) tot += vsum_s[q][c];
    tot *= kBf16Unscale;  // exact
    const float mu = smooth ? (float)(tot / (double)valid) : 0.0f;
    if (rg == 0) v_mean[((size_t)bh * T + b) * D + c] = mu;
    float vm[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    r = rg;
    for (; r + 3 * RG < valid; r += 4 * RG) {
#pragma unroll
        for (int e = 0; e < 4; ++e) vm[e] = fmaxf(vm[e], fabsf(__fsub_rn(bf2f(vsh[(r + e * RG) * D + c]), mu)));
    }
    for (; r < valid; r += RG) vm[0] = fmaxf(vm[0], fabsf(__fsub_rn(bf2f(vsh[r * D + c]), mu)));
    vmax_s[rg][c] = fmaxf(fmaxf(vm[0], vm[1]), fmaxf(vm[2], vm[3]));
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
// The block's gathered V rows are copied once, 16 bytes a piece, into shared
// memory; codes are built per channel and leave as 16-byte pieces of vt rows.
template <int D, int BK>
constexpr int v_quant_smem() {
    return BK * D * 2;
}

template <int D, int BK>
__global__ void __launch_bounds__(PREP_THREADS) prep_v_quant(const __nv_bfloat16* __restrict__ V,
                                                             const int32_t* __restrict__ perm, int smooth,
                                                             const float* __restrict__ v_mean,
                                                             const uint32_t* __restrict__ vamax,
                                                             uint8_t* __restrict__ vt_fp8, float* __restrict__ v_scale,
                                                             int N, int T, const int* __restrict__ status) {
    constexpr int NT = PREP_THREADS;
    constexpr int RG = NT / D;
    constexpr int CH = D / 8;
    constexpr int STRIDE = BK + 4;  // bytes per channel row of codes (conflict-free word stores)
    extern __shared__ uint4 v_s[];  // [BK][CH]
    __shared__ int tok_s[BK];
    __shared__ uint32_t cs[D * STRIDE / 4];
    if (ctl_failed(status)) return;  // perm is undefined
    const int b = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int valid = min(BK, N - b * BK);
    const int Tp = T * BK;
    for (int r = tid; r < BK; r += NT) tok_s[r] = r < valid ? clamp_tok(perm[(size_t)bh * N + b * BK + r], N) : 0;
    __syncthreads();
    const uint4* vg = reinterpret_cast<const uint4*>(V + (size_t)bh * N * D);
#pragma unroll
    for (int u = 0; u < BK * CH / NT; ++u) {
        const int i = tid + u * NT;
        const int r = i / CH;
        if (r < valid) cp_async16(v_s + i, vg + (size_t)tok_s[r] * CH + i % CH);
    }
    cp_async_wait_all();
    const int c = tid % D, rg = tid / D;
    const float amax = __uint_as_float(vamax[(size_t)bh * D + c]);
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
    if (b == 0 && rg == 0) v_scale[(size_t)bh * D + c] = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const float mu = v_mean[((size_t)bh * T + b) * D + c];
    __syncthreads();
    const __nv_bfloat16* vsh = reinterpret_cast<const __nv_bfloat16*>(v_s);
    for (int r4 = rg; r4 < BK / 4; r4 += RG) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = 4 * r4 + e;
            // padding tokens must be code 0 (x = +0 encodes to 0x00)
            x[e] = r < valid ? __fmul_rn(__fsub_rn(bf2f(vsh[r * D + c]), mu), inv) : 0.0f;
        }
        cs[(c * STRIDE) / 4 + r4] = (uint32_t)e4m3x2(x[0], x[1]) | ((uint32_t)e4m3x2(x[2], x[3]) << 16);
    }
    __syncthreads();
    constexpr int CHUNKS = BK / 16;
    for (int i = tid; i < D * CHUNKS; i += NT) {
        const int cc = i / CHUNKS, ch = i % CHUNKS;
        const uint32_t* src = cs + (cc * STRIDE) / 4 + ch * 4;
        *reinterpret_cast<uint4*>(vt_fp8 + ((size_t)bh * D + cc) * Tp + (size_t)b * BK + 16 * ch) =
            make_uint4(src[0], src[1], src[2], src[3]);
    }
}

// The 4-bit residual: the same block means and residual channel maxima as the
// E4M3 path, then per channel one fp32 scale s_c = amax_c/(6*448) and, for
// every 16 consecutive tokens of a channel inside the block, an NVFP4 block:
// y = r * (6*448/amax_c), UE4M3 scale E4M3(amax_16/6), codes E2M1(y * (1/s))
// (a zero scale codes zeros).  Codes leave transposed and packed two a byte
// (token 2i in the low nibble): vt[bh][c][token/2]; the block scales leave as
// v_bscale[bh][b][c][BK/16], the bytes one PV tile needs, contiguous.
template <int D, int BK>
__global__ void __launch_bounds__(PREP_THREADS) prep_v_quant_nvfp4(const __nv_bfloat16* __restrict__ V,
                                                                   const int32_t* __restrict__ perm,
                                                                   const float* __restrict__ v_mean,
                                                                   const uint32_t* __restrict__ vamax,
                                                                   uint8_t* __restrict__ vt_fp4,
                                                                   uint8_t* __restrict__ v_bscale,
                                                                   float* __restrict__ v_scale, int N, int T,
                                                                   const int* __restrict__ status) {
    constexpr int NT = PREP_THREADS;
    constexpr int RG = NT / D;
    constexpr int CH = D / 8;
    constexpr int G = BK / 16;       // NVFP4 blocks per channel and tile
    constexpr int WSTR = BK / 8 + 1; // words per channel row of codes (+1: conflict-free)
    extern __shared__ uint4 v_s[];   // [BK][CH]
    __shared__ int tok_s[BK];
    __shared__ uint32_t cw[D * WSTR];
    __shared__ __align__(16) uint8_t sc_s[D * G];  // read back as words
    if (ctl_failed(status)) return;  // perm is undefined
    const int b = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int valid = min(BK, N - b * BK);
    const int64_t Tp = (int64_t)T * BK;
    for (int r = tid; r < BK; r += NT) tok_s[r] = r < valid ? clamp_tok(perm[(size_t)bh * N + b * BK + r], N) : 0;
    __syncthreads();
    const uint4* vg = reinterpret_cast<const uint4*>(V + (size_t)bh * N * D);
#pragma unroll
    for (int u = 0; u < BK * CH / NT; ++u) {
        const int i = tid + u * NT;
        const int r = i / CH;
        if (r < valid) cp_async16(v_s + i, vg + (size_t)tok_s[r] * CH + i % CH);
    }
    cp_async_wait_all();
    const int c = tid % D, rg = tid / D;
    const float amax = __uint_as_float(vamax[(size_t)bh * D + c]);
    const float inv = amax > 0.0f ? __fdiv_rn(2688.0f, amax) : 0.0f;
    if (b == 0 && rg == 0) v_scale[(size_t)bh * D + c] = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    const float mu = v_mean[((size_t)bh * T + b) * D + c];
    __syncthreads();
    const __nv_bfloat16* vsh = reinterpret_cast<const __nv_bfloat16*>(v_s);
    for (int g = rg; g < G; g += RG) {
        float y[16];
        float ga = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int r = 16 * g + e;
            y[e] = r < valid ? __fmul_rn(__fsub_rn(bf2f(vsh[r * D + c]), mu), inv) : 0.0f;
            ga = fmaxf(ga, fabsf(y[e]));
        }
        const uint8_t sc = (uint8_t)(e4m3x2(__fdiv_rn(ga, 6.0f), 0.0f) & 0xFF);
        const float sv = e4m3_to_f32(sc);
        uint32_t w0 = 0, w1 = 0;
        if (sv > 0.0f) {
            const float rs = __frcp_rn(sv);
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = __fmul_rn(y[e], rs);
            w0 = e2m1x8(y);
            w1 = e2m1x8(y + 8);
        }
        cw[c * WSTR + 2 * g] = w0;
        cw[c * WSTR + 2 * g + 1] = w1;
        sc_s[c * G + g] = sc;
    }
    __syncthreads();
    // codes: BK/2 bytes a channel row, as 16-byte pieces
    constexpr int PIECES = BK / 32;
    for (int i = tid; i < D * PIECES; i += NT) {
        const int cc = i / PIECES, pc = i % PIECES;
        const uint32_t* src = cw + cc * WSTR + 4 * pc;
        *reinterpret_cast<uint4*>(vt_fp4 + ((size_t)bh * D + cc) * (Tp / 2) + (size_t)b * (BK / 2) + 16 * pc) =
            make_uint4(src[0], src[1], src[2], src[3]);
    }
    // block scales: D * G bytes, contiguous for the tile
    for (int i = tid; i < D * G / 4; i += NT)
        reinterpret_cast<uint32_t*>(v_bscale + ((size_t)bh * T + b) * D * G)[i] =
            reinterpret_cast<const uint32_t*>(sc_s)[i];
}

// Per-token Q: amax over d, inv = 448/amax, code = E4M3(q * inv), sq = amax/448.
// Per-token E4M3 Q: amax over the d channels, inv = 448/amax, code = E4M3(q *
// inv), scale = amax/448.  A token's row is read by D/8 lanes, 16 bytes each
// (amax over those lanes by xor shuffles), and every lane has four rows' loads
// in flight, so a warp covers 4 * 256/D tokens.
constexpr int QQ_TOK_PER_CTA = 8 * 4;  // warps x loads in flight, times 256/D tokens a load

template <int D>
__global__ void __launch_bounds__(256) quant_q(const __nv_bfloat16* __restrict__ Q, uint8_t* __restrict__ q_fp8,
                                               float* __restrict__ sq, int64_t tokens) {
    constexpr int LPT = D / 8;     // lanes per token
    constexpr int TPW = 32 / LPT;  // tokens a warp covers per load
    constexpr int U = 4;           // loads in flight per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPT, part = lane % LPT;
    const int64_t tok0 = ((int64_t)blockIdx.x * 8 + warp) * (TPW * U) + sub;
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t tok = tok0 + u * TPW;
        raw[u] = tok < tokens ? __ldg(reinterpret_cast<const uint4*>(Q + tok * D) + part) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t tok = tok0 + u * TPW;
        const uint32_t wd[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
        float x[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            x[2 * h] = __uint_as_float(wd[h] << 16);
            x[2 * h + 1] = __uint_as_float(wd[h] & 0xFFFF0000u);
        }
        float m = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
        for (int o = LPT / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float inv = m > 0.0f ? __fdiv_rn(448.0f, m) : 0.0f;
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
            w[h] = (uint32_t)e4m3x2(__fmul_rn(x[4 * h], inv), __fmul_rn(x[4 * h + 1], inv)) |
                   ((uint32_t)e4m3x2(__fmul_rn(x[4 * h + 2], inv), __fmul_rn(x[4 * h + 3], inv)) << 16);
        if (tok < tokens) {
            *reinterpret_cast<uint2*>(q_fp8 + tok * D + part * 8) = make_uint2(w[0], w[1]);
            if (part == 0) sq[tok] = __fdiv_rn(m, 448.0f);
        }
    }
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
    // Two CTAs share an SM when both fit in shared memory and TMEM (2 Cp columns
    // each); otherwise ask for enough shared memory to keep one CTA per SM, so
    // no CTA waits in tcgen05.alloc.
    // CTAs per SM: as many as shared memory (228 KB an SM) and TMEM (512
    // columns, 2 Cp a CTA) allow, at most three; the request is padded so no
    // more CTAs than that share an SM and none waits in tcgen05.alloc.
    const KmLayout lay(D, Cp);
    const int ncols = 2 * Cp <= 32 ? 32 : (2 * Cp <= 64 ? 64 : (2 * Cp <= 128 ? 128 : (2 * Cp <= 256 ? 256 : 512)));
    int cps = 3;
    while (cps > 1 && ((size_t)cps * lay.bytes > 227 * 1024 || cps * ncols > 512)) --cps;
    const size_t smem = lay.bytes > (size_t)(228 * 1024 / (cps + 1) + 1024) ? lay.bytes
                                                                             : (size_t)(228 * 1024 / (cps + 1) + 1024);
    // Tiles per CTA: about four waves of CTAs over the SMs.
    const int sms = sm_count();
    const int64_t tiles = (int64_t)nblk * p.BH;
    const int64_t slots = (int64_t)sms * cps * 4;
    const int tpc = (int)imin64(16, (tiles + slots - 1) / slots);
    const int nchunk = (nblk + tpc - 1) / tpc;
    static PerDeviceOnce configured;
    const int dev = PerDeviceOnce::current();
    if (!configured.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(km_assign<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(km_pass<D, 1, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(km_pass<D, 3, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(km_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, KM_SCAN_CHUNK * sizeof(int));
        if (e != cudaSuccess) return e;
        configured.mark(dev);
    }
    CUtensorMap tv, th, tl;
    if (!make_tmap_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.V, D, p.N, p.BH, 64, KM_TOK) ||
        !make_tmap_3d(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.c_hi, D, Cp, p.BH, 64, Cp) ||
        !make_tmap_3d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.c_lo, D, Cp, p.BH, 64, Cp))
        return cudaErrorInvalidValue;
    km_init<<<dim3(Cp, p.BH), D, 0, s>>>(p.V, p.c_hi, p.c_lo, p.cnorm, p.cent64, p.sums, p.state, p.vamax, p.tie_count, p.N, p.C,
                                         Cp, D);
    if (p.C <= 64) {
        // One fused pass a sweep (the member sums fit in shared memory); the
        // regroup is built once, from the last labels.
        using Sum = KpShape<1, 8>;   // passes 0 and 1: the update warps sum every token, then move the changed ones
        using Move = KpShape<3, 0>;  // later passes: atomics move the few changed tokens; the last pass
        const KpLayout ls(D, Cp, Sum::kStages, 1, Sum::kAcc, true), lm(D, Cp, Move::kStages, 3, Move::kAcc, false);
        const int grid = sms < KP_MAX_GRID ? sms : KP_MAX_GRID;
        int* regions = p.tie_count + 2;
        for (int it = 0; it < p.iters; ++it) {
            // pass 0 adds every token; pass 1 moves the tokens that change
            // (about a seventh of them) through the update warps, later passes
            // (a few per mille) with atomics; the last needs no sums
            const int mode = it + 1 == p.iters ? 0 : (it == 0 ? 1 : (it == 1 ? 3 : 2));
            if (mode == 1 || mode == 3)
                km_pass<D, 1, 8><<<grid, Sum::kThreads, ls.bytes, s>>>(tv, th, tl, p.cnorm, p.vnorm2, p.labels,
                                                                      p.hist, p.sums, p.ties, regions, p.state, p.BH,
                                                                      p.N, p.C, Cp, it, mode, p.ctl);
            else
                km_pass<D, 3, 0><<<grid, Move::kThreads, lm.bytes, s>>>(tv, th, tl, p.cnorm, p.vnorm2, p.labels,
                                                                       p.hist, p.sums, p.ties, regions, p.state, p.BH,
                                                                       p.N, p.C, Cp, it, mode, p.ctl);
            km_refine<D><<<sms * 8, 256, 0, s>>>(p.ties, p.tie_count, regions, grid, p.c_hi, p.c_lo, p.cnorm,
                                                  p.V, p.cent64, p.labels,
                                                  p.hist, p.sums, p.state, p.N, p.C, Cp, it, mode != 0,
                                                  p.ctl.status);
            if (mode != 0)  // the sums stay: every later pass moves changed tokens only
                km_finalize<<<dim3(p.C, p.BH), D, 0, s>>>(p.c_hi, p.c_lo, p.cnorm, p.cent64, p.sums, p.ccount,
                                                          p.hist, p.state, p.C, Cp, D, nblk, it, 1, 1,
                                                          p.ctl.status);
        }
        km_scan<<<p.BH, 1024, KM_SCAN_CHUNK * sizeof(int), s>>>(p.hist, p.offs, p.cstart, p.ccount, p.state, p.N,
                                                                 p.C, nblk, p.iters - 1, 0, p.ctl.status);
        km_scatter<<<dim3(nblk, p.BH), KM_TOK, 0, s>>>(p.labels, p.offs, p.perm, p.state, p.N, p.C, 0,
                                                       p.ctl.status);
        return cudaGetLastError();
    }
    for (int it = 0; it < p.iters; ++it) {
        km_assign<D><<<dim3(nchunk, p.BH), 128, smem, s>>>(tv, th, tl, p.cnorm, p.cent64, p.V, p.vnorm2, p.labels,
                                                            p.hist, p.ties, p.tie_count, p.state, p.N, p.C, Cp,
                                                            it, tpc, p.ctl);
        km_refine<D><<<sms * 8, 256, 0, s>>>(p.ties, p.tie_count, nullptr, 0, p.c_hi, p.c_lo, p.cnorm, p.V,
                                              p.cent64, p.labels, p.hist,
                                              p.sums, p.state, p.N, p.C, Cp, it, 0, p.ctl.status);
        km_scan<<<p.BH, 1024, KM_SCAN_CHUNK * sizeof(int), s>>>(p.hist, p.offs, p.cstart, p.ccount, p.state, p.N,
                                                                 p.C, nblk, it, 1, p.ctl.status);
        km_scatter<<<dim3(nblk, p.BH), KM_TOK, 0, s>>>(p.labels, p.offs, p.perm, p.state, p.N, p.C, 1,
                                                       p.ctl.status);
        if (it + 1 < p.iters) {
            km_update<D><<<dim3((p.N + KM_UPD_ROWS - 1) / KM_UPD_ROWS, p.BH), 128, 0, s>>>(
                p.V, p.perm, p.cstart, p.sums, p.state, p.N, p.C, p.ctl.status);
            km_finalize<<<dim3(p.C, p.BH), D, 0, s>>>(p.c_hi, p.c_lo, p.cnorm, p.cent64, p.sums, p.ccount, p.hist,
                                                      p.state, p.C, Cp, D, nblk, it, 0, 0, p.ctl.status);
        }
    }
    return cudaGetLastError();
}

template <int D, int BK>
static cudaError_t blocks_t(const PrepLaunch& p, cudaStream_t s) {
    const int T = (p.N + BK - 1) / BK;
    if (p.smooth != 1) {  // no k-means this call: the channel maxima start from zero here
        if (p.smooth == 0) {  // plain per-channel FP8 V: identity order
            const int64_t total = (int64_t)p.BH * p.N;
            identity_order<<<(unsigned)imin64((total + 255) / 256, 32LL * sm_count()), 256, 0, s>>>(p.perm, p.labels,
                                                                                                 total, p.N);
        }  // smooth == 2: the regroup already in perm is kept
        cudaError_t e = cudaMemsetAsync(p.vamax, 0, sizeof(uint32_t) * (size_t)p.BH * D, s);
        if (e != cudaSuccess) return e;
    }
    static PerDeviceOnce configured;
    const int dev = PerDeviceOnce::current();
    if (!configured.done(dev)) {
        cudaError_t e = cudaFuncSetAttribute(prep_kv_block<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kv_block_smem<D, BK>());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(prep_v_quant<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 v_quant_smem<D, BK>());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(prep_v_quant_nvfp4<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 v_quant_smem<D, BK>());
        if (e != cudaSuccess) return e;
        configured.mark(dev);
    }
    prep_kv_block<D, BK><<<dim3(T, p.BH), PREP_THREADS, kv_block_smem<D, BK>(), s>>>(
        p.K, p.V, p.perm, p.smooth, p.k_fp8, p.k_scale, p.v_mean, p.vamax, p.N, T, p.ctl.status);
    if (p.resid_fmt == 1) {
        if constexpr (BK % 32 == 0) {
            prep_v_quant_nvfp4<D, BK><<<dim3(T, p.BH), PREP_THREADS, v_quant_smem<D, BK>(), s>>>(
                p.V, p.perm, p.v_mean, p.vamax, p.vt_fp8, p.v_bscale, p.v_scale, p.N, T, p.ctl.status);
        }
    } else {
        prep_v_quant<D, BK><<<dim3(T, p.BH), PREP_THREADS, v_quant_smem<D, BK>(), s>>>(
            p.V, p.perm, p.smooth, p.v_mean, p.vamax, p.vt_fp8, p.v_scale, p.N, T, p.ctl.status);
    }
    return cudaGetLastError();
}

cudaError_t launch_prep(const PrepLaunch& p, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    if (p.smooth == 1) {
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
    const int64_t per_cta = QQ_TOK_PER_CTA * 256 / D;  // 32 tokens a CTA at d 128, 64 at d 64
    const unsigned grid = (unsigned)((tokens + per_cta - 1) / per_cta);
    if (D == 128)
        quant_q<128><<<grid, 256, 0, s>>>(Q, q_fp8, sq, tokens);
    else
        quant_q<64><<<grid, 256, 0, s>>>(Q, q_fp8, sq, tokens);
    return cudaGetLastError();
}

cudaError_t launch_e4m3_encode(const float* x, uint8_t* out, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const unsigned grid = (unsigned)imin64((n + 255) / 256, 16LL * sm_count());
    e4m3_encode_kernel<<<grid, 256, 0, s>>>(x, out, n);
    return cudaGetLastError();
}

}  // namespace vc
