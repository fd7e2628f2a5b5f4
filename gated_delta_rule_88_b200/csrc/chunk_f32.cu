// chunk_f32.cu -- exact-fp32 chunkwise KDA prefill (SIMT, no tensor cores).
//
// Serves fp32 inputs, where the tolerance is an absolute 1e-3 and bf16
// tensor-core operands would not do, and bf16 inputs at head dimensions the
// tensor-core kernels do not take (dk or dv = 64): the bf16 values are
// widened on load, every step is fp32, and the output is rounded to nearest
// even on store.  It is the chunkwise form of the Kimi
// Linear paper notes, section 3: within a chunk of C = 64 tokens the old
// state's contribution goes through the chunk's transitions and the
// intra-chunk writes are gathered by a WY-like transform.  With G the
// chunk-local inclusive cumsum of g (per channel) and, for tokens i, j of the
// chunk,
//     A_ij = beta_i sum_c k_ic k_jc exp(G_ic - G_jc)   (j < i)
//     P_ij =        sum_c q_ic k_jc exp(G_ic - G_jc)   (j <= i)
//     T    = (I + A)^-1                     (unit lower triangular)
//     V_new = T [beta (V - (K e^G) S)]      (the u_t of the recurrence)
//     O     = (Q e^G) S + P V_new
//     S    <- Diag(e^{G_C}) S + (K e^{G_C - G})^T V_new
// Each exp(G_ic - G_jc) is taken per element (j <= i, so its argument is the
// decay between the two tokens and never overflows for g <= 0): exact and
// robust, affordable because this path only serves fp32 inputs.
//
// One CTA per (sequence, head, 32-column dv tile) walks its chunks in order;
// the intra-chunk part is recomputed per dv tile.  Partial last chunks are
// padded with q = k = v = g = beta = 0, which leaves every real row unchanged
// and makes G_C the cumsum at the last real token.
#include "common.cuh"
#include "kernels.h"

namespace kda {

namespace {

constexpr int CH = 64;        // chunk length
constexpr int DVT = 32;       // dv columns per CTA
constexpr int NT = 256;
constexpr int LDA = CH + 1;   // padded 64x64 matrices

template <int DK>
struct F32Smem {
    static constexpr int LD = DK + 1;           // padded rows of q, k, G
    float Qs[CH * LD];      // q, then q e^G
    float Ks[CH * LD];      // k, then k e^{G_C - G}
    float Gs[CH * LD];      // G, then k e^G
    float Vs[CH * DVT];     // v tile, then V_new
    float Xs[CH * DVT];     // beta (V - (K e^G) S)
    float Ss[DK * DVT];     // state tile S[c][n]
    float Am[CH * LDA];     // A, then (Q e^G) S
    float Tm[CH * LDA];     // T
    float Pm[CH * LDA];     // P
    float bs[CH];
    float eGC[DK];          // exp(G_C)
    float GC[DK];           // G_C, the cumsum at the chunk's last row
};

// TI: the type of q, k, v and out (float or __nv_bfloat16)
template <int DK, typename TI>
__global__ void __launch_bounds__(NT)
chunk_f32_kernel(const TI *__restrict__ q, const TI *__restrict__ k,
                 const TI *__restrict__ v, const float *__restrict__ g,
                 const float *__restrict__ beta, const float *__restrict__ s0,
                 const int32_t *__restrict__ cu, TI *__restrict__ out,
                 float *__restrict__ sT, int T, int total_T, int H, int dv, Prologue pro)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    F32Smem<DK> &sm = *reinterpret_cast<F32Smem<DK> *>(smem_raw);
    constexpr int LD = F32Smem<DK>::LD;

    const int tid = threadIdx.x;
    const int n0 = blockIdx.x * DVT;   // first dv column of this tile
    const int h = blockIdx.y;
    const int seq = blockIdx.z;

    long long bos, eos;
    if (cu) {
        bos = min(max(cu[seq], 0), total_T);
        eos = min(max(cu[seq + 1], 0), total_T);
        if (eos < bos) eos = bos;
    } else {
        bos = (long long)seq * T;
        eos = bos + T;
    }

    // initial state tile
    const size_t sbase = ((size_t)seq * H + h) * (size_t)DK * dv;
    for (int i = tid; i < DK * DVT; i += NT) {
        const int c = i / DVT, n = i % DVT;
        sm.Ss[i] = s0 ? s0[sbase + (size_t)c * dv + n0 + n] : 0.f;
    }

    for (long long t0 = bos; t0 < eos; t0 += CH) {
        const int len = (int)min((long long)CH, eos - t0);
        __syncthreads();   // previous chunk fully consumed

        // ---- load the chunk (zero padding past the end) ----
        for (int i = tid; i < CH * DK; i += NT) {
            const int r = i / DK, c = i % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (r < len) {
                const size_t off = ((size_t)(t0 + r) * H + h) * DK + c;
                qv = to_f(q[off]); kv = to_f(k[off]); gv = g[off];
            }
            sm.Qs[r * LD + c] = qv; sm.Ks[r * LD + c] = kv; sm.Gs[r * LD + c] = gv;
        }
        for (int i = tid; i < CH * DVT; i += NT) {
            const int r = i / DVT, n = i % DVT;
            sm.Vs[i] = (r < len) ? to_f(v[((size_t)(t0 + r) * H + h) * dv + n0 + n]) : 0.f;
        }
        if (tid < CH) {
            float bt = (tid < len) ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
            if ((pro.flags & kProBetaSigmoid) && tid < len) bt = sigmoid_f(bt);
            sm.bs[tid] = bt;
        }
        __syncthreads();
        // ---- prologue: row factors of q (with q_scale) and k ----
        if (pro.flags != 0 || pro.q_scale != 1.f) {
            for (int rr = tid; rr < 2 * CH; rr += NT) {
                float *row = rr < CH ? &sm.Qs[rr * LD] : &sm.Ks[(rr - CH) * LD];
                float f = 1.f;
                if (pro.flags & kProQkL2Norm) {
                    float ss = 0.f;
                    for (int c = 0; c < DK; ++c) ss = fmaf(row[c], row[c], ss);
                    f = inv_norm(ss);
                }
                if (rr < CH) f *= pro.q_scale;
                for (int c = 0; c < DK; ++c) row[c] *= f;
            }
            __syncthreads();
        }

        // ---- G: chunk-local inclusive cumsum of g per channel ----
        if (tid < DK) {
            float acc = 0.f;
            for (int r = 0; r < CH; ++r) { acc += sm.Gs[r * LD + tid]; sm.Gs[r * LD + tid] = acc; }
            sm.GC[tid] = acc;
            sm.eGC[tid] = expf(acc);
        }
        __syncthreads();

        // ---- A (strict lower) and P (lower incl. diagonal), per element ----
        for (int p = tid; p < CH * (CH + 1) / 2; p += NT) {
            int i = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
            while (i * (i + 1) / 2 > p) --i;
            while ((i + 1) * (i + 2) / 2 <= p) ++i;
            const int j = p - i * (i + 1) / 2;
            float a = 0.f, pp = 0.f;
            const float *qi = &sm.Qs[i * LD], *ki = &sm.Ks[i * LD], *kj = &sm.Ks[j * LD];
            const float *gi = &sm.Gs[i * LD], *gj = &sm.Gs[j * LD];
#pragma unroll 4
            for (int c = 0; c < DK; ++c) {
                const float e = expf(gi[c] - gj[c]);
                const float kje = kj[c] * e;
                a += ki[c] * kje;
                pp += qi[c] * kje;
            }
            sm.Am[i * LDA + j] = (j < i) ? sm.bs[i] * a : 0.f;
            sm.Pm[i * LDA + j] = pp;
        }
        __syncthreads();

        // ---- T = (I + A)^-1 by forward substitution, one column per thread ----
        if (tid < CH) {
            const int c = tid;
            for (int i = 0; i < c; ++i) sm.Tm[i * LDA + c] = 0.f;
            sm.Tm[c * LDA + c] = 1.f;
            for (int i = c + 1; i < CH; ++i) {
                float acc = 0.f;
                for (int j = c; j < i; ++j) acc += sm.Am[i * LDA + j] * sm.Tm[j * LDA + c];
                sm.Tm[i * LDA + c] = -acc;
            }
        }
        __syncthreads();

        // ---- decayed forms: Q e^G, K e^G, K e^{G_C - G} ----
        for (int i = tid; i < CH * DK; i += NT) {
            const int r = i / DK, c = i % DK;
            const float G = sm.Gs[r * LD + c];
            const float kv = sm.Ks[r * LD + c];
            const float eG = expf(G);
            sm.Qs[r * LD + c] *= eG;
            sm.Ks[r * LD + c] = kv * expf(sm.GC[c] - G);
            sm.Gs[r * LD + c] = kv * eG;
        }
        __syncthreads();

        // ---- X = beta (V - (K e^G) S), Y = (Q e^G) S ----
        {
            const int n = tid % DVT;
            for (int i = tid / DVT; i < CH; i += NT / DVT) {
                float x = 0.f, y = 0.f;
                for (int c = 0; c < DK; ++c) {
                    const float s = sm.Ss[c * DVT + n];
                    x += sm.Gs[i * LD + c] * s;
                    y += sm.Qs[i * LD + c] * s;
                }
                sm.Xs[i * DVT + n] = sm.bs[i] * (sm.Vs[i * DVT + n] - x);
                sm.Am[i * LDA + n] = y;
            }
        }
        __syncthreads();

        // ---- V_new = T X ----
        {
            const int n = tid % DVT;
            for (int i = tid / DVT; i < CH; i += NT / DVT) {
                float acc = 0.f;
                for (int j = 0; j <= i; ++j) acc += sm.Tm[i * LDA + j] * sm.Xs[j * DVT + n];
                sm.Vs[i * DVT + n] = acc;
            }
        }
        __syncthreads();

        // ---- O = Y + P V_new ; S <- Diag(e^{G_C}) S + (K e^{G_C-G})^T V_new ----
        {
            const int n = tid % DVT;
            for (int i = tid / DVT; i < len; i += NT / DVT) {
                float acc = sm.Am[i * LDA + n];
                for (int j = 0; j <= i; ++j) acc += sm.Pm[i * LDA + j] * sm.Vs[j * DVT + n];
                out[((size_t)(t0 + i) * H + h) * dv + n0 + n] = from_f<TI>(acc);
            }
            for (int c = tid / DVT; c < DK; c += NT / DVT) {
                float acc = sm.eGC[c] * sm.Ss[c * DVT + n];
                for (int i = 0; i < CH; ++i) acc += sm.Ks[i * LD + c] * sm.Vs[i * DVT + n];
                sm.Ss[c * DVT + n] = acc;
            }
        }
    }
    __syncthreads();
    if (sT) {
        for (int i = tid; i < DK * DVT; i += NT) {
            const int c = i / DVT, n = i % DVT;
            sT[sbase + (size_t)c * dv + n0 + n] = sm.Ss[i];
        }
    }
}

template <int DK, typename TI>
cudaError_t launch_chunk_f32_t(const TI *q, const TI *k, const TI *v, const float *g,
                               const float *beta, const float *s0, const int32_t *cu,
                               TI *out, float *sT, int N, int T, int total_T, int H,
                               int dv, Prologue pro, cudaStream_t st)
{
    const size_t smem = sizeof(F32Smem<DK>);
    cudaError_t e = cudaFuncSetAttribute(chunk_f32_kernel<DK, TI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(dv / DVT, H, N);
    chunk_f32_kernel<DK, TI><<<grid, NT, smem, st>>>(q, k, v, g, beta, s0, cu, out, sT, T,
                                                     total_T, H, dv, pro);
    return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *s0, const int32_t *cu, void *out,
                              float *sT, int N, int T, int total_T, int H, int dk, int dv,
                              Prologue pro, cudaStream_t st)
{
    if (dv % DVT != 0) return cudaErrorInvalidValue;
    const TI *q_ = (const TI *)q, *k_ = (const TI *)k, *v_ = (const TI *)v;
    if (dk == 64)
        return launch_chunk_f32_t<64, TI>(q_, k_, v_, g, beta, s0, cu, (TI *)out, sT, N, T, total_T, H, dv, pro, st);
    if (dk == 128)
        return launch_chunk_f32_t<128, TI>(q_, k_, v_, g, beta, s0, cu, (TI *)out, sT, N, T, total_T, H, dv, pro, st);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_chunk_f32(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *s0, const int32_t *cu,
                             void *out, float *sT, int N, int T, int total_T, int H,
                             int dk, int dv, bool bf16, Prologue pro, cudaStream_t st)
{
    return bf16 ? launch_chunk_simt<__nv_bfloat16>(q, k, v, g, beta, s0, cu, out, sT, N, T, total_T, H, dk, dv, pro, st)
                : launch_chunk_simt<float>(q, k, v, g, beta, s0, cu, out, sT, N, T, total_T, H, dk, dv, pro, st);
}

}  // namespace kda
