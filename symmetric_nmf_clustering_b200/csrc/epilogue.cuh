// The per-tile epilogue of an S-stream pass, in two forms: epilogue_tile (128
// threads, the standalone epilogue kernel of the CUDA-core path and of the
// passes without a stream) and epilogue_tile_cta (all 256 threads of the last
// split CTA of each 128-row tile in the tensor-core stream kernel).
//
// For the rows i of one tile, with P_i = sum over splits of the partial rows
// (fixed split order), by mode:
//   FULL        tr partial sum_c H_ic P_ic; g = 4 (H_i A - P_i);
//               G' = G + g*g; H' = max(H - lr g / (sqrt(G') + eps), 0)
//               ([CaS] "Factorizing with SymNMF"; [SMI] AdaptGrow sketch);
//               Gram partial of H'; exact TF32 split of H' for the next pass
//   SNAPSHOT    P~_i = P_i; tr partial (Block-SVRG snapshot)
//   SVRG_INNER  P_i <- P~_i + m Y_i, then the FULL step without the trace
//   STEP_SNAP   P_i <- P~_i, then the FULL step without the trace
//   GRAM        Gram partial of H (and its TF32 split)
//   PRODUCT     Y_i = P_i
#pragma once

#include "common.cuh"

namespace symnmf {

constexpr int EP_ROWS = 128;

// 16-byte global -> shared copy that bypasses L1 (the data were written by
// other CTAs of the same kernel), and the wait for all of this thread's copies
__device__ __forceinline__ void cp_async_cg16(float* dst_smem, const float* src) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst_smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

struct EpiArgs {
    int mode;
    int64_t n;
    int k;
    const float* part;     // splits x n x k partial products
    int splits;
    const float* H;
    const float* G;
    float* Hn;
    float* Gn;
    float* Psnap;
    float m_scale, lr, eps;
    double* tr_part;       // one per tile
    double* gram_part;     // k*k per tile
    float* Y;
    const FitState* st;
    float* XT;             // split operand of the rows left in h (may be null)
    int64_t ldxt;
    float* hmax_part;      // FULL / GRAM: max |h| over the tile's rows left in h (may be null)
};

// Max over the threads of a block of `nt` threads (a multiple of 32); the
// result is valid in every thread.  wred: nt / 32 floats of shared memory.
__device__ __forceinline__ float ep_block_max(float v, int tid, int nt, float* wred) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((tid & 31) == 0) wred[tid >> 5] = v;
    __syncthreads();
    float m = 0.f;
    for (int w = 0; w < nt / 32; ++w) m = fmaxf(m, wred[w]);
    __syncthreads();
    return m;
}

// The evaluation's scalar step (one thread): f_t = ||S||^2 - 2 tr + ||A||^2,
// history, relative change, stopping test ([CaS] "Factorizing with SymNMF";
// the trace identity of "Factorization at scale").
__device__ __forceinline__ void finalize_scalar(int mode, FitState* st, double tr, double rel_tol,
                                                int max_evals, double* history, int history_cap) {
    const bool eval = mode == MODE_FULL || mode == MODE_SNAPSHOT;
    const int t = st->t;
    bool stop = false;
    if (eval) {
        const double L = st->s_sqnorm - 2.0 * tr + st->a_sqnorm;
        if (t < history_cap && history != nullptr) history[t] = L;
        if (!isfinite(L)) {
            st->nonfinite = 1;
            stop = true;
        }
        if (t > 0) {
            const double Lp = st->loss;
            double rel;
            if (Lp != 0.0) rel = fabs(L - Lp) / fabs(Lp);
            else rel = (L == Lp) ? 0.0 : INFINITY;
            st->rel = rel;
            if (rel_tol > 0.0 && rel < rel_tol) {
                st->converged = 1;
                stop = true;
            }
        }
        st->loss_prev = st->loss;
        st->loss = L;
        st->t_stop = t;
        if (t >= max_evals - 1) stop = true;
        st->t = t + 1;
    }
    if (stop) st->done = 1;
}



// Fixed-shape sum over the 128 threads (warp shuffles, then warp 0); the
// result is valid in tid 0.
__device__ __forceinline__ double ep_sum(double v, int tid, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    const int w = tid >> 5, l = tid & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = 0.0;
    if (w == 0) {
        r = l < EP_ROWS / 32 ? red[l] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r += __shfl_down_sync(0xffffffffu, r, o);
    }
    __syncthreads();
    return r;
}

// smem: at least max(KE*KE, EP_ROWS*(KE+1)) floats; red: EP_ROWS/32 doubles.
template <int KE>
__device__ void epilogue_tile(const EpiArgs& a, int tile, int tid, float* smem, double* red) {
    const int mode = a.mode;
    const int64_t n = a.n;
    const int k = a.k;
    float* As = smem;                                            // k x k Gram (step modes)
    float(*hs)[KE + 1] = reinterpret_cast<float(*)[KE + 1]>(smem);  // rows for the Gram partial

    const int64_t i = (int64_t)tile * EP_ROWS + tid;
    const bool valid = i < n;
    const bool step = mode == MODE_FULL || mode == MODE_SVRG_INNER || mode == MODE_STEP_SNAP;

    if (step) {
        for (int e = tid; e < k * k; e += EP_ROWS) As[(e / k) * KE + (e % k)] = a.st->A32[e];
        __syncthreads();
    }

    float p[KE], h[KE];
#pragma unroll
    for (int c = 0; c < KE; ++c) {
        p[c] = 0.f;
        h[c] = 0.f;
    }
    if (valid) {
        const int64_t row = i * (int64_t)k;
        if (mode != MODE_GRAM && mode != MODE_STEP_SNAP) {
            for (int s = 0; s < a.splits; ++s) {
                const float* src = a.part + (int64_t)s * n * k + row;
#pragma unroll
                for (int c = 0; c < KE; ++c)
                    if (c < k) p[c] += __ldcg(src + c);   // written by other CTAs
            }
        }
        if (mode == MODE_STEP_SNAP) {
#pragma unroll
            for (int c = 0; c < KE; ++c)
                if (c < k) p[c] = a.Psnap[row + c];
        } else if (mode == MODE_SVRG_INNER) {
#pragma unroll
            for (int c = 0; c < KE; ++c)
                if (c < k) p[c] = fmaf(a.m_scale, p[c], a.Psnap[row + c]);
        }
        if (mode == MODE_PRODUCT) {
#pragma unroll
            for (int c = 0; c < KE; ++c)
                if (c < k) a.Y[row + c] = p[c];
            return;
        }
        if (mode == MODE_SNAPSHOT) {
#pragma unroll
            for (int c = 0; c < KE; ++c)
                if (c < k) a.Psnap[row + c] = p[c];
        }
#pragma unroll
        for (int c = 0; c < KE; ++c)
            if (c < k) h[c] = a.H[row + c];
    }
    if (mode == MODE_PRODUCT) return;

    // trace partial: sum_i sum_c H_ic (S H)_ic in fp64 (products of fp32 are exact)
    if (mode == MODE_FULL || mode == MODE_SNAPSHOT) {
        double tr = 0.0;
#pragma unroll
        for (int c = 0; c < KE; ++c) tr += (double)h[c] * (double)p[c];
        const double tot = ep_sum(tr, tid, red);
        if (tid == 0) a.tr_part[tile] = tot;
    }
    if (mode == MODE_SNAPSHOT) return;

    if (step && valid) {
        const int64_t row = i * (int64_t)k;
        float hnew[KE];
#pragma unroll
        for (int c = 0; c < KE; ++c) {
            hnew[c] = 0.f;
            if (c < k) {
                float ha = 0.f;
#pragma unroll
                for (int d = 0; d < KE; ++d)
                    if (d < k) ha = fmaf(h[d], As[d * KE + c], ha);
                const float g = 4.f * (ha - p[c]);
                const float gg = fmaf(g, g, a.G[row + c]);
                const float stepv = __fdiv_rn(a.lr * g, __fadd_rn(__fsqrt_rn(gg), a.eps));
                hnew[c] = fmaxf(h[c] - stepv, 0.f);
                a.Gn[row + c] = gg;
                a.Hn[row + c] = hnew[c];
            }
        }
#pragma unroll
        for (int c = 0; c < KE; ++c) h[c] = hnew[c];
    }

    // exact TF32 split [h_hi; h_lo] of the rows in h, the next S-stream's operand
    if (a.XT != nullptr && valid &&
        (mode == MODE_FULL || mode == MODE_STEP_SNAP || mode == MODE_GRAM)) {
        const int KP = (k + 7) / 8 * 8;
#pragma unroll
        for (int c = 0; c < KE; ++c) {
            if (c < k) {
                const float hb = __uint_as_float(__float_as_uint(h[c]) & 0xFFFFE000u);
                a.XT[(int64_t)c * a.ldxt + i] = hb;
                a.XT[(int64_t)(KP + c) * a.ldxt + i] = h[c] - hb;
            }
        }
    }

    if (a.hmax_part != nullptr && (mode == MODE_FULL || mode == MODE_GRAM)) {
        __shared__ float wred[EP_ROWS / 32];
        float m = 0.f;
#pragma unroll
        for (int c = 0; c < KE; ++c)
            if (valid && c < k) m = fmaxf(m, fabsf(h[c]));
        m = ep_block_max(m, tid, EP_ROWS, wred);
        if (tid == 0) a.hmax_part[tile] = m;
    }

    // Gram partial of the rows now in h (new iterate, or the given H for GRAM)
    __syncthreads();  // every thread is done reading As
#pragma unroll
    for (int c = 0; c < KE; ++c) hs[tid][c] = valid ? h[c] : 0.f;
    __syncthreads();
    const int rows = (int)min64(EP_ROWS, n - (int64_t)tile * EP_ROWS);
    double* gp = a.gram_part + (int64_t)tile * k * k;
    for (int e = tid; e < k * k; e += EP_ROWS) {
        const int c = e / k, d = e % k;
        // four interleaved chains (fixed order), combined as ((s0 + s1) + (s2 + s3))
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        int r = 0;
        for (; r + 4 <= rows; r += 4) {
            s0 = fma((double)hs[r][c], (double)hs[r][d], s0);
            s1 = fma((double)hs[r + 1][c], (double)hs[r + 1][d], s1);
            s2 = fma((double)hs[r + 2][c], (double)hs[r + 2][d], s2);
            s3 = fma((double)hs[r + 3][c], (double)hs[r + 3][d], s3);
        }
        for (; r < rows; ++r) s0 = fma((double)hs[r][c], (double)hs[r][d], s0);
        gp[e] = (s0 + s1) + (s2 + s3);
    }
}

}  // namespace symnmf

namespace symnmf {

// Shared-memory floats epilogue_tile_cta<KE> needs (tiles, Gram, reduction).
template <int KE>
constexpr size_t epilogue_cta_floats() {
    return 3 * (size_t)EP_ROWS * KE + (size_t)KE * KE + 32;
}

// The same per-tile epilogue, run by all 256 threads of one CTA (the last
// split CTA of the tile in the tensor-core stream kernel).  Global loads and
// stores are coalesced through shared-memory tiles; each element sees the
// same arithmetic as epilogue_tile (partials summed in split order, H A
// accumulated in d order, the same AdaGrad expression), and each Gram entry
// the same four-chain fp64 sum (products of fp32 values are exact in fp64, so
// entry (c, d) equals entry (d, c) and is computed once).  The trace partial
// is summed in a different, fixed order.
// smem: stage_floats >= epilogue_cta_floats<KE>() floats, 16-byte aligned.
// Callers: every thread of the CTA.
template <int KE>
__device__ void epilogue_tile_cta(const EpiArgs& a, int tile, int tid, float* smem, int stage_floats) {
    constexpr int NT = 256;
    static_assert(EP_ROWS * KE % NT == 0, "whole elements per thread");
    const int mode = a.mode;
    const int64_t n = a.n;
    const int k = a.k;
    const int64_t i0 = (int64_t)tile * EP_ROWS;
    const int rows = (int)min64(EP_ROWS, n - i0);
    const int tot = rows * k;                       // elements of the tile, row-major, stride k
    const int64_t base = i0 * (int64_t)k;
    float* P = smem;                                // [EP_ROWS * KE] partial sums
    float* T2 = P + EP_ROWS * KE;                   // G, then G'
    float* T1 = T2 + EP_ROWS * KE;                  // H, then H'
    float* As = T1 + EP_ROWS * KE;                  // k x k Gram of the iterate
    double* red = reinterpret_cast<double*>(As + KE * KE);   // 16 doubles
    double* Hd = reinterpret_cast<double*>(P);      // H' in fp64 (row stride KE + 2), aliases P, T2, T1
    const bool step = mode == MODE_FULL || mode == MODE_SVRG_INNER || mode == MODE_STEP_SNAP;

    // ---- stage the tile: P = sum of partials (or the snapshot product), H, G, A.
    // Thread tid owns elements tid + q*NT (q < EPT).  Every global load is
    // issued before the first shared-memory store (the compiler cannot tell the
    // two address spaces apart through these pointers), and each split's loads
    // for all of a thread's elements go out together, so the tile costs about
    // one L2 round trip per split (per two splits when registers allow).
    constexpr int EPT = EP_ROWS * KE / NT;
    constexpr int AEL = (KE * KE + NT - 1) / NT;
    const bool snap_in = mode == MODE_STEP_SNAP || mode == MODE_SVRG_INNER;
    float ps[EPT], hv[EPT], gv[EPT], av[AEL];
    if (mode != MODE_PRODUCT) {
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = tid + q * NT;
            const bool in = e < tot;
            ps[q] = (in && snap_in) ? __ldcg(a.Psnap + base + e) : 0.f;
            hv[q] = in ? __ldcg(a.H + base + e) : 0.f;
            gv[q] = (in && step) ? __ldcg(a.G + base + e) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < AEL; ++q) {
            const int e = tid + q * NT;
            av[q] = (step && e < k * k) ? a.st->A32[e] : 0.f;
        }
    }
    float acc[EPT];
#pragma unroll
    for (int q = 0; q < EPT; ++q) acc[q] = 0.f;
    // the partial tiles are contiguous runs of 16-byte pieces when n k and the
    // tile's element count are multiples of 4: they then go to shared memory
    // (all of it is free until P, H, G and A are stored below) with cp.async,
    // as many tiles per batch as fit, one L2 round trip per batch
    constexpr int TS = EP_ROWS * KE;
    const int nbt = stage_floats / TS;
    const bool staged = nbt >= 1 && (n * k) % 4 == 0 && tot % 4 == 0;
    if (staged && mode != MODE_GRAM && mode != MODE_STEP_SNAP) {
        for (int s0 = 0; s0 < a.splits; s0 += nbt) {
            const int sb = min(nbt, a.splits - s0);
            for (int t = 0; t < sb; ++t) {
                const float* src = a.part + (int64_t)(s0 + t) * n * k + base;
                for (int e4 = tid; e4 < tot / 4; e4 += NT)
                    cp_async_cg16(smem + t * TS + 4 * e4, src + 4 * e4);
            }
            cp_async_wait_all();
            __syncthreads();
            for (int t = 0; t < sb; ++t) {
#pragma unroll
                for (int q = 0; q < EPT; ++q) {
                    const int e = tid + q * NT;
                    if (e < tot) acc[q] += smem[t * TS + e];
                }
            }
            __syncthreads();   // read before the next batch (or P, H, G) overwrites
        }
    } else if (mode != MODE_GRAM && mode != MODE_STEP_SNAP) {
        int s = 0;
        if constexpr (EPT <= 16) {
            for (; s + 1 < a.splits; s += 2) {
                const float* s0 = a.part + (int64_t)s * n * k + base;
                const float* s1 = s0 + n * k;
                float v0[EPT], v1[EPT];
#pragma unroll
                for (int q = 0; q < EPT; ++q) {
                    const int e = tid + q * NT;
                    v0[q] = e < tot ? __ldcg(s0 + e) : 0.f;
                    v1[q] = e < tot ? __ldcg(s1 + e) : 0.f;
                }
#pragma unroll
                for (int q = 0; q < EPT; ++q) {
                    acc[q] += v0[q];
                    acc[q] += v1[q];
                }
            }
        }
        for (; s < a.splits; ++s) {
            const float* src = a.part + (int64_t)s * n * k + base;
            float v[EPT];
#pragma unroll
            for (int q = 0; q < EPT; ++q) {
                const int e = tid + q * NT;
                v[q] = e < tot ? __ldcg(src + e) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < EPT; ++q) acc[q] += v[q];
        }
    }
    if (mode == MODE_PRODUCT) {
#pragma unroll
        for (int q = 0; q < EPT; ++q) {
            const int e = tid + q * NT;
            if (e < tot) a.Y[base + e] = acc[q];
        }
        return;
    }
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
        const int e = tid + q * NT;
        if (e >= tot) continue;
        float p = acc[q];
        if (mode == MODE_STEP_SNAP) p = ps[q];
        else if (mode == MODE_SVRG_INNER) p = fmaf(a.m_scale, p, ps[q]);
        if (mode == MODE_SNAPSHOT) a.Psnap[base + e] = p;
        P[e] = p;
        T1[e] = hv[q];
        if (step) T2[e] = gv[q];
    }
    if (step) {
#pragma unroll
        for (int q = 0; q < AEL; ++q) {
            const int e = tid + q * NT;
            if (e < k * k) As[(e / k) * KE + (e % k)] = av[q];
        }
    }
    __syncthreads();

    // ---- trace partial sum_i sum_c H_ic P_ic (fp64; fp32 products are exact)
    if (mode == MODE_FULL || mode == MODE_SNAPSHOT) {
        double tr = 0.0;
        for (int e = tid; e < tot; e += NT) tr += (double)T1[e] * (double)P[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tr += __shfl_down_sync(0xffffffffu, tr, o);
        if ((tid & 31) == 0) red[tid >> 5] = tr;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int w = 0; w < NT / 32; ++w) t += red[w];
            a.tr_part[tile] = t;
        }
    }
    if (mode == MODE_SNAPSHOT) return;

    // ---- projected AdaGrad step: two threads per row, KE/2 columns each
    if (step) {
        constexpr int HALF = KE / 2;   // a multiple of 4
        const int r = tid >> 1, c0 = (tid & 1) * HALF;
        float hn[HALF], gn[HALF];
        const bool valid = r < rows;
        if ((k & 3) == 0) {
            // rows of H, P, G and of A read as 16-byte pieces (r k, c0 and KE
            // are multiples of 4), H A accumulated in the same d order
            float h[KE], ha[HALF];
#pragma unroll
            for (int m = 0; m < KE / 4; ++m) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (valid && 4 * m < k) x = *reinterpret_cast<const float4*>(T1 + r * k + 4 * m);
                h[4 * m] = x.x;
                h[4 * m + 1] = x.y;
                h[4 * m + 2] = x.z;
                h[4 * m + 3] = x.w;
            }
#pragma unroll
            for (int j = 0; j < HALF; ++j) ha[j] = 0.f;
#pragma unroll
            for (int d = 0; d < KE; ++d) {
                if (d < k) {
#pragma unroll
                    for (int m = 0; m < HALF / 4; ++m) {
                        const float4 a4 = *reinterpret_cast<const float4*>(As + d * KE + c0 + 4 * m);
                        ha[4 * m] = fmaf(h[d], a4.x, ha[4 * m]);
                        ha[4 * m + 1] = fmaf(h[d], a4.y, ha[4 * m + 1]);
                        ha[4 * m + 2] = fmaf(h[d], a4.z, ha[4 * m + 2]);
                        ha[4 * m + 3] = fmaf(h[d], a4.w, ha[4 * m + 3]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < HALF / 4; ++m) {
                float4 p4 = make_float4(0.f, 0.f, 0.f, 0.f), g4 = p4, h4 = p4;
                if (valid && c0 + 4 * m < k) {
                    p4 = *reinterpret_cast<const float4*>(P + r * k + c0 + 4 * m);
                    g4 = *reinterpret_cast<const float4*>(T2 + r * k + c0 + 4 * m);
                    h4 = *reinterpret_cast<const float4*>(T1 + r * k + c0 + 4 * m);
                }
                const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
                const float gv4[4] = {g4.x, g4.y, g4.z, g4.w};
                const float hv4[4] = {h4.x, h4.y, h4.z, h4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = 4 * m + u;
                    hn[j] = 0.f;
                    gn[j] = 0.f;
                    if (valid && c0 + j < k) {
                        const float g = 4.f * (ha[j] - pv[u]);
                        const float gg = fmaf(g, g, gv4[u]);
                        const float stepv = __fdiv_rn(a.lr * g, __fadd_rn(__fsqrt_rn(gg), a.eps));
                        hn[j] = fmaxf(hv4[u] - stepv, 0.f);
                        gn[j] = gg;
                    }
                }
            }
        } else {
            float h[KE];
#pragma unroll
            for (int d = 0; d < KE; ++d) h[d] = (valid && d < k) ? T1[r * k + d] : 0.f;
#pragma unroll
            for (int j = 0; j < HALF; ++j) {
                const int c = c0 + j;
                hn[j] = 0.f;
                gn[j] = 0.f;
                if (valid && c < k) {
                    float ha = 0.f;
#pragma unroll
                    for (int d = 0; d < KE; ++d)
                        if (d < k) ha = fmaf(h[d], As[d * KE + c], ha);
                    const float g = 4.f * (ha - P[r * k + c]);
                    const float gg = fmaf(g, g, T2[r * k + c]);
                    const float stepv = __fdiv_rn(a.lr * g, __fadd_rn(__fsqrt_rn(gg), a.eps));
                    hn[j] = fmaxf(T1[r * k + c] - stepv, 0.f);   // = h[c]
                    gn[j] = gg;
                }
            }
        }
        __syncthreads();   // every thread holds its row of H: T1, T2 may be overwritten
        if (valid) {
#pragma unroll
            for (int j = 0; j < HALF; ++j) {
                const int c = c0 + j;
                if (c < k) {
                    T1[r * k + c] = hn[j];
                    T2[r * k + c] = gn[j];
                }
            }
        }
        __syncthreads();
        for (int e = tid; e < tot; e += NT) {
            a.Hn[base + e] = T1[e];
            a.Gn[base + e] = T2[e];
        }
    }

    // ---- exact TF32 split [h_hi; h_lo] of the rows now in T1 (the next pass's operand)
    if (a.XT != nullptr && (mode == MODE_FULL || mode == MODE_STEP_SNAP || mode == MODE_GRAM)) {
        const int KP = (k + 7) / 8 * 8;
        for (int e = tid; e < k * EP_ROWS; e += NT) {
            const int c = e / EP_ROWS, r = e % EP_ROWS;
            if (r < rows) {
                const float v = T1[r * k + c];
                const float hb = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
                a.XT[(int64_t)c * a.ldxt + i0 + r] = hb;
                a.XT[(int64_t)(KP + c) * a.ldxt + i0 + r] = v - hb;
            }
        }
    }

    // ---- Gram partial of the rows in T1, in fp64.  The rows go through
    // registers so that Hd (row stride KE + 2: 16-byte aligned, and eight
    // consecutive rows fall in distinct banks) can overwrite P, T2 and T1.
    constexpr int HS = KE + 2;
    static_assert(EP_ROWS * HS * 2 <= 3 * EP_ROWS * KE, "Hd fits in P, T2 and T1");
    __syncthreads();
    float hreg[EPT];
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
        const int e = tid + q * NT, r = e / KE, c = e % KE;
        hreg[q] = (r < rows && c < k) ? T1[r * k + c] : 0.f;
    }
    if (a.hmax_part != nullptr && (mode == MODE_FULL || mode == MODE_GRAM)) {
        __shared__ float wred[NT / 32];
        float m = 0.f;
#pragma unroll
        for (int q = 0; q < EPT; ++q) m = fmaxf(m, fabsf(hreg[q]));
        m = ep_block_max(m, tid, NT, wred);
        if (tid == 0) a.hmax_part[tile] = m;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
        const int e = tid + q * NT, r = e / KE, c = e % KE;
        Hd[r * HS + c] = (double)hreg[q];
    }
    __syncthreads();
    // 4x4 register blocks of the upper triangle; the rows of the tile are cut
    // into RG groups whose partial blocks sit in adjacent lanes and are
    // combined by a fixed xor-shuffle tree (every lane ends with the same sum)
    constexpr int NB = KE / 4, NBLK = NB * (NB + 1) / 2;
    constexpr int RG = NBLK * 32 <= NT ? 32 : NBLK * 16 <= NT ? 16 : NBLK * 8 <= NT ? 8
                     : NBLK * 4 <= NT ? 4 : NBLK * 2 <= NT ? 2 : 1;
    constexpr int RROWS = EP_ROWS / RG;   // rows grp, grp + RG, grp + 2 RG, ...
    static_assert(NBLK * RG <= NT && 32 % RG == 0, "one Gram task per thread, groups inside a warp");
    double gacc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) gacc[i][j] = 0.0;
    const int blk = tid / RG, grp = tid % RG;
    int bi = 0, bj = 0;
    if (blk < NBLK) {
        int rem = blk;
        while (rem >= NB - bi) {
            rem -= NB - bi;
            ++bi;
        }
        bj = bi + rem;
        // rows past the tile's end hold zeros, which add exactly nothing
        for (int t = 0; t < RROWS; ++t) {
            const double* hr = Hd + (grp + t * RG) * HS;
            const double2 x01 = *reinterpret_cast<const double2*>(hr + 4 * bi);
            const double2 x23 = *reinterpret_cast<const double2*>(hr + 4 * bi + 2);
            const double2 y01 = *reinterpret_cast<const double2*>(hr + 4 * bj);
            const double2 y23 = *reinterpret_cast<const double2*>(hr + 4 * bj + 2);
            const double x[4] = {x01.x, x01.y, x23.x, x23.y};
            const double y[4] = {y01.x, y01.y, y23.x, y23.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) gacc[i][j] = fma(x[i], y[j], gacc[i][j]);
        }
    }
#pragma unroll
    for (int o = 1; o < RG; o <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) gacc[i][j] += __shfl_xor_sync(0xffffffffu, gacc[i][j], o);
    if (blk < NBLK && grp == 0) {
        double* gp = a.gram_part + (int64_t)tile * k * k;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = 4 * bi + i, d = 4 * bj + j;
                if (c < k && d < k) {
                    gp[c * k + d] = gacc[i][j];
                    gp[d * k + c] = gacc[i][j];
                }
            }
    }
}

}  // namespace symnmf

