/*
 * frt_oracle.c -- plain, slow, obviously-correct CPU oracle for the fused
 * static-FP8 attention-input chain.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the timed CPU
 * baseline of the benchmark use it.  It shares no source with the CUDA
 * library (no headers, no helpers, no tables); it is compiled by gcc on its
 * own, with -ffp-contract=off so that every a*b+c below is two roundings,
 * exactly as written.
 *
 * Citations name the page of the flashrt-structures 0.2.0 wheel that the
 * step follows and the symbol on it:
 *   [qkv_pack]   impls/qkv_pack/fp8_static.py          (wheel page 34)
 *   [ptok_table] impls/modnorm_qkv_chain/fp8_ptok_table.py (wheel page 30)
 *   [fp8_chain]  impls/adarms_stack/fp8_chain.py        (wheel page 16)
 *
 * Arithmetic is fp32 (the pages do every step in `.float()`), except the
 * rotary angle and its cos/sin, which are fp64 and rounded once to bf16.
 * Every accumulation runs in index order.  Where the pages are silent the
 * reading taken is stated at the function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bf16: the 16 high bits of an IEEE binary32.                          */
/* ------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float or_bf16_to_f32(uint16_t h) { return f32_from_bits(((uint32_t)h) << 16); }

/* Round a binary32 to bf16, nearest with ties to even.  The 16 dropped
 * bits are compared with one half-unit (0x8000) of the kept last place. */
uint16_t or_bf16_from_f32(float f)
{
    uint32_t u = bits_from_f32(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

/* Round a binary64 to bf16 once (no intermediate binary32 rounding):
 * bracket |d| between the two bf16 neighbours and take the nearer one,
 * ties to the even code.  Used for the cos/sin table only (|d| <= 1). */
uint16_t or_bf16_from_f64(double d)
{
    if (d == 0.0) return signbit(d) ? 0x8000u : 0u;
    double a = fabs(d);
    float t = (float)a;
    if ((double)t > a) t = nextafterf(t, 0.0f);       /* truncate toward 0 */
    uint32_t lo_code = bits_from_f32(t) >> 16;         /* bf16 below |d| */
    double lo = (double)f32_from_bits(lo_code << 16);
    double hi = (double)f32_from_bits((lo_code + 1u) << 16);
    uint32_t code;
    if (a == lo) code = lo_code;
    else {
        double mid = 0.5 * (lo + hi);                  /* exact in binary64 */
        if (a < mid) code = lo_code;
        else if (a > mid) code = lo_code + 1u;
        else code = (lo_code & 1u) ? lo_code + 1u : lo_code;
    }
    return (uint16_t)(code | (signbit(d) ? 0x8000u : 0u));
}

/* ------------------------------------------------------------------ */
/* float8 e4m3fn: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no inf; */
/* S.1111.111 is NaN, so the largest finite magnitude is 1.75*2^8=448.  */
/* ------------------------------------------------------------------ */

float or_e4m3_to_f32(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    float mag;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) mag = (float)m * ldexpf(1.0f, -9);            /* subnormal */
    else mag = (1.0f + (float)m / 8.0f) * ldexpf(1.0f, e - 7); /* normal */
    return s ? -mag : mag;
}

/* Quantize the way the pages write it, `(v).clamp(-448, 448).to(e4m3fn)`
 * ([qkv_pack] _pack_weights; [ptok_table] _q8): clamp first, then round to
 * the nearest representable magnitude, ties to the even code (mantissa
 * LSB 0), the sign kept (tiny negatives give 0x80).  The search runs over
 * the 127 finite non-negative codes, which are ordered by value. */
uint8_t or_e4m3_from_f32(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (a > 448.0f) a = 448.0f;
    int lo = 0, hi = 0x7E;                 /* invariant: val(lo) <= a <= val(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (or_e4m3_to_f32((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    float vlo = or_e4m3_to_f32((uint8_t)lo), vhi = or_e4m3_to_f32((uint8_t)hi);
    int code;
    if (a <= vlo) code = lo;
    else if (a >= vhi) code = hi;
    else {
        float half = 0.5f * (vlo + vhi);   /* exact: few significant bits */
        if (a < half) code = lo;
        else if (a > half) code = hi;
        else code = (lo & 1) ? hi : lo;
    }
    return (uint8_t)(sign | code);
}

/* q8(v; s) = e4m3(clamp(v / s)) with a true fp32 division. */
static uint8_t q8(float v, float s) { return or_e4m3_from_f32(v / s); }

/* ------------------------------------------------------------------ */
/* Producer, AdaRMS form ([fp8_chain] norm_project and the final tail). */
/* ------------------------------------------------------------------ */
/*
 * Per row r, columns j (all fp32):
 *   h      = res[r,j] + g[r|0,j] * delta[r,j]     gated residual add
 *   res   <- bf16(h)                              stored in place
 *   ms     = (sum_j bf16(h)^2) / D                over the stored residual
 *   inv    = 1 / sqrt(ms + eps)                   eps inside the root
 *   y      = ((bf16(h) * inv) * w_j) * (1 + scale_j) + shift_j
 *   x8     = q8(y; act_scale)
 *   gate_out[r,j] = gate_j
 * Style chunk order is (scale, shift, gate): the stack's tail applies
 * `normed * (1 + fin[0]) + fin[1]` and the style stack documents one
 * (scale, shift, gate) projection per norm.
 * Readings (the pages are silent): the norm is taken over the bf16-rounded
 * residual, the value the next layer sees; weight multiplies before the
 * modulation; no rounding between the steps of y.
 * weight == NULL means ones (the chain passes a ones vector).
 * gate_stride / style_stride are row strides in elements; 0 broadcasts
 * row 0 to every row.  y_out (rows*D fp32) and amax_out are optional.
 */
void or_ada_rms_norm_quant(int rows, int D, float eps,
                           uint16_t *res, const uint16_t *delta,
                           const uint16_t *prev_gate, long gate_stride,
                           const uint16_t *weight,
                           const uint16_t *style, long style_stride,
                           float act_scale, uint8_t *x8, uint16_t *gate_out,
                           float *y_out, float *amax_out)
{
    float *row_amax = (float *)calloc((size_t)(rows > 0 ? rows : 1), sizeof(float));
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        uint16_t *rr = res + (size_t)r * D;
        const uint16_t *dd = delta + (size_t)r * D;
        const uint16_t *gg = prev_gate + (size_t)r * gate_stride;
        const uint16_t *st = style + (size_t)r * style_stride;
        float ss = 0.0f;
        for (int j = 0; j < D; ++j) {
            float h = or_bf16_to_f32(rr[j]) + or_bf16_to_f32(gg[j]) * or_bf16_to_f32(dd[j]);
            rr[j] = or_bf16_from_f32(h);
            float hr = or_bf16_to_f32(rr[j]);
            ss = ss + hr * hr;
        }
        float ms = ss / (float)D;
        float inv = 1.0f / sqrtf(ms + eps);
        float mx = 0.0f;
        for (int j = 0; j < D; ++j) {
            float hr = or_bf16_to_f32(rr[j]);
            float w = weight ? or_bf16_to_f32(weight[j]) : 1.0f;
            float scale = or_bf16_to_f32(st[j]);
            float shift = or_bf16_to_f32(st[D + j]);
            float t = hr * inv;
            t = t * w;
            t = t * (1.0f + scale);
            float y = t + shift;
            x8[(size_t)r * D + j] = q8(y, act_scale);
            if (y_out) y_out[(size_t)r * D + j] = y;
            if (fabsf(y) > mx) mx = fabsf(y);
            if (gate_out) gate_out[(size_t)r * D + j] = st[2 * D + j];
        }
        row_amax[r] = mx;
    }
    if (amax_out) {
        float mx = 0.0f;
        for (int r = 0; r < rows; ++r) if (row_amax[r] > mx) mx = row_amax[r];
        *amax_out = mx;
    }
    free(row_amax);
}

/* ------------------------------------------------------------------ */
/* Producer, per-token-table LayerNorm form ([ptok_table]               */
/* PerTokenModChainBlock.forward and the producer bind smoke).          */
/* ------------------------------------------------------------------ */
/*
 * Per token r (all fp32):
 *   shift_j = table[shift_idx, j] + temb[r, shift_idx, j]
 *   scale_j = table[scale_idx, j] + temb[r, scale_idx, j]
 *   mu      = (sum_j x_j) / D
 *   var     = (sum_j (x_j - mu)^2) / D          biased, two passes
 *   y       = ((x_j - mu) * (1 / sqrt(var + eps))) * (1 + scale_j) + shift_j
 *   x8      = q8(y; act_scale)
 * The block table's chunk order is (shift, scale, gate) per site; the
 * attention site passes (0, 1), the FFN site (3, 4).  The LayerNorm has
 * no affine weight.  Reading: the modulation is (1 + scale) * x + shift,
 * the same form the AdaRMS tail uses.  The gate is not produced here.
 */
void or_ada_layer_norm_quant_table(int rows, int D, float eps,
                                   const uint16_t *x, const uint16_t *temb,
                                   int chunks, const float *table,
                                   int shift_idx, int scale_idx,
                                   float act_scale, uint8_t *x8,
                                   float *y_out, float *amax_out)
{
    float *row_amax = (float *)calloc((size_t)(rows > 0 ? rows : 1), sizeof(float));
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const uint16_t *xr = x + (size_t)r * D;
        const uint16_t *tr = temb + (size_t)r * chunks * D;
        float sum = 0.0f;
        for (int j = 0; j < D; ++j) sum = sum + or_bf16_to_f32(xr[j]);
        float mu = sum / (float)D;
        float sq = 0.0f;
        for (int j = 0; j < D; ++j) {
            float c = or_bf16_to_f32(xr[j]) - mu;
            sq = sq + c * c;
        }
        float var = sq / (float)D;
        float inv = 1.0f / sqrtf(var + eps);
        float mx = 0.0f;
        for (int j = 0; j < D; ++j) {
            float shift = table[(size_t)shift_idx * D + j] + or_bf16_to_f32(tr[(size_t)shift_idx * D + j]);
            float scale = table[(size_t)scale_idx * D + j] + or_bf16_to_f32(tr[(size_t)scale_idx * D + j]);
            float t = (or_bf16_to_f32(xr[j]) - mu) * inv;
            t = t * (1.0f + scale);
            float y = t + shift;
            x8[(size_t)r * D + j] = q8(y, act_scale);
            if (y_out) y_out[(size_t)r * D + j] = y;
            if (fabsf(y) > mx) mx = fabsf(y);
        }
        row_amax[r] = mx;
    }
    if (amax_out) {
        float mx = 0.0f;
        for (int r = 0; r < rows; ++r) if (row_amax[r] > mx) mx = row_amax[r];
        *amax_out = mx;
    }
    free(row_amax);
}

/* ------------------------------------------------------------------ */
/* Joint per-tensor weight pack ([qkv_pack] _pack_weights; the chain's  */
/* _quantize with _interleave_rows).                                    */
/* ------------------------------------------------------------------ */
/*
 * Siblings w_i [n_i, K] (bf16) are stacked along N.  One scale for the
 * whole stack: s = max(amax(|w|) / 448, 1e-8); w8 = q8(w; s).  Missing
 * biases are zeros (bias_i == NULL).  `layout` only permutes rows:
 *   0  plain concatenation (the pages' torch.cat order);
 *   1  q/k head interleave: in every head of siblings 0 and 1 (q, k),
 *      source row i < hd/2 goes to 2i and row hd/2 + i goes to 2i + 1, so
 *      an adjacent-pair rotation carries the host's rotate-half rotation;
 *      sibling 2 (v) keeps host order.  The map is the inverse of the
 *      chain's `kperm` (kperm[2i] = i, kperm[2i+1] = hd/2 + i).
 * Any other layout value is treated as 0.
 */
static long pack_dest_row(int layout, int sib, long i, long base, int hd)
{
    if (layout == 1 && (sib == 0 || sib == 1)) {
        long head = i / hd, d = i % hd, half = hd / 2;
        long dst = d < half ? 2 * d : 2 * (d - half) + 1;
        return base + head * hd + dst;
    }
    return base + i;
}

void or_pack_weights_fp8(int n_sib, const uint16_t *const *w, const int *n_i,
                         int K, const uint16_t *const *bias, int layout,
                         int hd, uint8_t *w8_out, float *w_scale_out,
                         uint16_t *bias_out)
{
    float amax = 0.0f;
    for (int s = 0; s < n_sib; ++s)
        for (long e = 0; e < (long)n_i[s] * K; ++e) {
            float a = fabsf(or_bf16_to_f32(w[s][e]));
            if (a > amax) amax = a;
        }
    float scale = amax / 448.0f;
    if (scale < 1e-8f) scale = 1e-8f;
    *w_scale_out = scale;
    long base = 0;
    for (int s = 0; s < n_sib; ++s) {
        /* rows are quantized independently (one shared scale) */
        #pragma omp parallel for schedule(static)
        for (long i = 0; i < n_i[s]; ++i) {
            long dst = pack_dest_row(layout, s, i, base, hd);
            for (int k = 0; k < K; ++k)
                w8_out[dst * K + k] = q8(or_bf16_to_f32(w[s][i * K + k]), scale);
            if (bias_out)
                bias_out[dst] = (bias && bias[s]) ? bias[s][i] : (uint16_t)0;
        }
        base += n_i[s];
    }
}

/* ------------------------------------------------------------------ */
/* Packed FP8 GEMM ([qkv_pack] PackedLinear._run; [fp8_chain]           */
/* norm_project: alpha = act_scale * w_scale).                          */
/* ------------------------------------------------------------------ */
/*
 * Y[m, n] = bf16( (sum_k x8[m,k] * w8[n,k]) * alpha + bias[n] ),
 * alpha = act_scale * w_scale in fp32; the sum is fp32 in k order (each
 * e4m3 x e4m3 product is exact in fp32); bias (bf16, optional) is added
 * after the scaling; one bf16 rounding at the end.  Rows are independent:
 * `row_index` (optional) lists which rows of x8 to compute, the result for
 * the i-th listed row going to out row i.  ldo is out's row stride.
 */
void or_fp8_gemm(int M, int N, int K, const uint8_t *x8, const uint8_t *w8,
                 float act_scale, float w_scale, const uint16_t *bias,
                 uint16_t *out, long ldo, const int *row_index, int n_rows)
{
    float dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = or_e4m3_to_f32((uint8_t)c);
    float alpha = act_scale * w_scale;
    int rows = row_index ? n_rows : M;
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < rows; ++i) {
        long m = row_index ? row_index[i] : i;
        const uint8_t *xr = x8 + m * (long)K;
        float *xf = (float *)malloc(sizeof(float) * (size_t)K);
        for (int k = 0; k < K; ++k) xf[k] = dec[xr[k]];
        for (int n = 0; n < N; ++n) {
            const uint8_t *wr = w8 + (long)n * K;
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) acc = acc + xf[k] * dec[wr[k]];
            float y = acc * alpha;
            if (bias) y = y + or_bf16_to_f32(bias[n]);
            out[(long)i * ldo + n] = or_bf16_from_f32(y);
        }
        free(xf);
    }
}

/* ------------------------------------------------------------------ */
/* Rotary table ([fp8_chain] _build_rope).                               */
/* ------------------------------------------------------------------ */
/*
 * rope[s, 2i] = bf16(cos(p * theta^(-2i/hd))), rope[s, 2i+1] = bf16(sin(..)),
 * p = P + s, i < hd/2.  The pages read cos/sin from the host's rotary
 * module and keep the first half (the half-duplicated form); reading: the
 * standard inverse-frequency formula, evaluated in fp64, rounded once.
 */
void or_rope_table(int M, int hd, int P, double theta, uint16_t *rope)
{
    int half = hd / 2;
    for (int s = 0; s < M; ++s)
        for (int i = 0; i < half; ++i) {
            double inv_freq = pow(theta, -(double)(2 * i) / (double)hd);
            double ang = (double)(P + s) * inv_freq;
            rope[(long)s * hd + 2 * i] = or_bf16_from_f64(cos(ang));
            rope[(long)s * hd + 2 * i + 1] = or_bf16_from_f64(sin(ang));
        }
}

/* ------------------------------------------------------------------ */
/* Split + RoPE + KV write ([fp8_chain] _make_run, the split kernel's   */
/* call, and _alloc for the buffer layouts).                             */
/* ------------------------------------------------------------------ */
/*
 * qkv [B*M, (hq + 2*hkv)*hd] bf16, row b*M + s.  For q and k heads, each
 * adjacent pair (x0, x1) = (x[2i], x[2i+1]) with c = rope[s,2i],
 * sn = rope[s,2i+1] becomes (x0*c - x1*sn, x0*sn + x1*c) in fp32, rounded
 * to bf16.  q goes to q_out [B, M, hq, hd]; k and v (v copied) go to the
 * caches [B, T, hkv, hd] at row P + s.  Nothing else of the caches is
 * touched.
 */
void or_split_rope_kvcache(int B, int M, int hq, int hkv, int hd, int P, int T,
                           const uint16_t *qkv, const uint16_t *rope,
                           uint16_t *q_out, uint16_t *k_cache, uint16_t *v_cache)
{
    long N = (long)(hq + 2 * hkv) * hd;
    for (int b = 0; b < B; ++b)
        for (int s = 0; s < M; ++s) {
            const uint16_t *row = qkv + ((long)b * M + s) * N;
            const uint16_t *rp = rope + (long)s * hd;
            for (int h = 0; h < hq + hkv; ++h) {
                const uint16_t *src = row + (long)h * hd;
                uint16_t *dst = h < hq
                    ? q_out + (((long)b * M + s) * hq + h) * hd
                    : k_cache + (((long)b * T + P + s) * hkv + (h - hq)) * hd;
                for (int i = 0; i < hd / 2; ++i) {
                    float x0 = or_bf16_to_f32(src[2 * i]);
                    float x1 = or_bf16_to_f32(src[2 * i + 1]);
                    float c = or_bf16_to_f32(rp[2 * i]);
                    float sn = or_bf16_to_f32(rp[2 * i + 1]);
                    float o0 = x0 * c - x1 * sn;
                    float o1 = x0 * sn + x1 * c;
                    dst[2 * i] = or_bf16_from_f32(o0);
                    dst[2 * i + 1] = or_bf16_from_f32(o1);
                }
            }
            for (int h = 0; h < hkv; ++h) {
                const uint16_t *src = row + (long)(hq + hkv + h) * hd;
                uint16_t *dst = v_cache + (((long)b * T + P + s) * hkv + h) * hd;
                for (int d = 0; d < hd; ++d) dst[d] = src[d];
            }
        }
}

/*
 * Prefix copy ([fp8_chain] _make_run, the `ad:prefix` range): the host
 * cache holds k, v as [B, hkv, T_src, hd]; rows p < P go to the chain's
 * caches [B, T, hkv, hd].  With `interleave`, the key's head dimension is
 * gathered through kperm (kperm[2i] = i, kperm[2i+1] = hd/2 + i) so the
 * host's rotate-half keys land in the adjacent-pair layout; v is copied.
 */
void or_prefix_copy(int B, int hkv, int hd, int P, int T, int T_src,
                    const uint16_t *prefix_k, const uint16_t *prefix_v,
                    int interleave, uint16_t *k_cache, uint16_t *v_cache)
{
    for (int b = 0; b < B; ++b)
        for (int p = 0; p < P; ++p)
            for (int h = 0; h < hkv; ++h) {
                const uint16_t *ks = prefix_k + (((long)b * hkv + h) * T_src + p) * hd;
                const uint16_t *vs = prefix_v + (((long)b * hkv + h) * T_src + p) * hd;
                uint16_t *kd = k_cache + (((long)b * T + p) * hkv + h) * hd;
                uint16_t *vd = v_cache + (((long)b * T + p) * hkv + h) * hd;
                for (int d = 0; d < hd; ++d) {
                    int src = interleave ? (d % 2 == 0 ? d / 2 : hd / 2 + d / 2) : d;
                    kd[d] = ks[src];
                    vd[d] = vs[d];
                }
            }
}

/* ------------------------------------------------------------------ */
/* Merged GEGLU + static requant ([fp8_chain] down_project; the bind   */
/* requires a tanh-approximate GELU).                                   */
/* ------------------------------------------------------------------ */
/*
 * gu [M, 2H] bf16 holds gate in columns [0, H) and up in [H, 2H).
 *   gelu_tanh(g) = 0.5 * g * (1 + tanh(sqrt(2/pi) * (g + 0.044715 * g^3)))
 *   hid8[m, j]   = q8(gelu_tanh(g) * u; out_scale)
 * all in fp32 (tanhf from the C library).
 */
void or_geglu_quant(int M, int H, const uint16_t *gu, float out_scale,
                    uint8_t *hid8, float *amax_out)
{
    const float k0 = 0.7978845608028654f;   /* sqrt(2/pi) */
    const float k1 = 0.044715f;
    float *row_amax = (float *)calloc((size_t)(M > 0 ? M : 1), sizeof(float));
    #pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        float mx = 0.0f;
        for (int j = 0; j < H; ++j) {
            float g = or_bf16_to_f32(gu[(long)m * 2 * H + j]);
            float u = or_bf16_to_f32(gu[(long)m * 2 * H + H + j]);
            float g3 = (g * g) * g;
            float inner = k0 * (g + k1 * g3);
            float gl = (0.5f * g) * (1.0f + tanhf(inner));
            float h = gl * u;
            hid8[(long)m * H + j] = q8(h, out_scale);
            if (fabsf(h) > mx) mx = fabsf(h);
        }
        row_amax[m] = mx;
    }
    if (amax_out) {
        float mx = 0.0f;
        for (int m = 0; m < M; ++m) if (row_amax[m] > mx) mx = row_amax[m];
        *amax_out = mx;
    }
    free(row_amax);
}

/* ------------------------------------------------------------------ */
/* Static quantize of the attention output ([fp8_chain] `out_project`: */
/* quantize_fp8_static_bf16(att2, t_sc_o) before the o_proj GEMM).      */
/* ------------------------------------------------------------------ */
/*
 *   x8[r, j] = q8(x[r, j]; scale)        x bf16 [rows, D], row stride ldx
 *   amax     = max |x|                   (the calibration statistic)
 */
void or_quant_fp8_static(int rows, int D, const uint16_t *x, long ldx, float scale,
                         uint8_t *x8, float *amax_out)
{
    float mx = 0.0f;
    for (int r = 0; r < rows; ++r) {
        for (int j = 0; j < D; ++j) {
            float v = or_bf16_to_f32(x[(long)r * ldx + j]);
            x8[(long)r * D + j] = q8(v, scale);
            if (fabsf(v) > mx) mx = fabsf(v);
        }
    }
    if (amax_out) *amax_out = mx;
}

/* ------------------------------------------------------------------ */
/* Final AdaRMS tail of the stack ([fp8_chain] `_make_run`, the         */
/* "ad:tail" range after the layer loop).                               */
/* ------------------------------------------------------------------ */
/*
 * Per row r, all fp32 (the page lifts res, gate and delta to fp32 and does
 * not round the sum to bf16 before the norm):
 *   h_j   = res_j + gate_j * delta_j
 *   ms    = (sum_j h_j^2) / D
 *   out_j = bf16((h_j * (1 / sqrt(ms + eps))) * (1 + fin[0, j]) + fin[1, j])
 * fin: fp32 rows (scale, shift) of the last norm, fin_stride elements apart
 * (the page keeps them fp32: they are sliced from the fp32 projection
 * before the bf16 cast of the styles).  gate_stride 0 broadcasts one gate
 * row.  The page writes torch.rsqrt; the reading here is 1 / sqrt, the
 * same as the producer's.
 */
void or_ada_rms_tail(int rows, int D, float eps, const uint16_t *res,
                     const uint16_t *delta, const uint16_t *gate, long gate_stride,
                     const float *fin, long fin_stride, uint16_t *out)
{
    float *h = (float *)malloc((size_t)(D > 0 ? D : 1) * sizeof(float));
    for (int r = 0; r < rows; ++r) {
        const uint16_t *rr = res + (long)r * D;
        const uint16_t *dd = delta + (long)r * D;
        const uint16_t *gg = gate + (long)r * gate_stride;
        float ss = 0.0f;
        for (int j = 0; j < D; ++j) {
            h[j] = or_bf16_to_f32(rr[j]) + or_bf16_to_f32(gg[j]) * or_bf16_to_f32(dd[j]);
            ss = ss + h[j] * h[j];
        }
        float ms = ss / (float)D;
        float inv = 1.0f / sqrtf(ms + eps);
        for (int j = 0; j < D; ++j) {
            float t = h[j] * inv;
            t = t * (1.0f + fin[j]);
            out[(long)r * D + j] = or_bf16_from_f32(t + fin[fin_stride + j]);
        }
    }
    free(h);
}

/* ------------------------------------------------------------------ */
/* GELU + static requant between the DiT FFN's two GEMMs ([ptok_table] */
/* PerTokenModChainBlock.forward: the fp8_gelu_mlp call on the FFN      */
/* site's FP8 activation, with the ffn_hid static scale).               */
/* ------------------------------------------------------------------ */
/*
 * u [M, H] bf16 (the up projection's bf16 output, bias included):
 *   hid8[m, j] = q8(gelu_tanh(u[m, j]); out_scale)
 * gelu_tanh as in or_geglu_quant (the kernel's GELU variant is not shown on
 * the pages; the tanh form is the reading), fp32, tanhf from the C library.
 */
void or_gelu_quant(int M, int H, const uint16_t *u, long ldu, float out_scale,
                   uint8_t *hid8, float *amax_out)
{
    const float k0 = 0.7978845608028654f;   /* sqrt(2/pi) */
    const float k1 = 0.044715f;
    float *row_amax = (float *)calloc((size_t)(M > 0 ? M : 1), sizeof(float));
    #pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        float mx = 0.0f;
        for (int j = 0; j < H; ++j) {
            float g = or_bf16_to_f32(u[(long)m * ldu + j]);
            float g3 = (g * g) * g;
            float inner = k0 * (g + k1 * g3);
            float h = (0.5f * g) * (1.0f + tanhf(inner));
            hid8[(long)m * H + j] = q8(h, out_scale);
            if (fabsf(h) > mx) mx = fabsf(h);
        }
        row_amax[m] = mx;
    }
    if (amax_out) {
        float mx = 0.0f;
        for (int m = 0; m < M; ++m) if (row_amax[m] > mx) mx = row_amax[m];
        *amax_out = mx;
    }
    free(row_amax);
}

/* ------------------------------------------------------------------ */
/* Modulation projection ([fp8_chain] _style_stack, and the per-step    */
/* table bake in the binder: one stacked dense projection of the        */
/* conditioning vector gives every norm its (scale, shift, gate)).      */
/* ------------------------------------------------------------------ */
/*
 * st[r, n] = sum_k cond[r, k] * w[n, k] + bias[n]
 * in fp32 (the binder runs addmm on `.float()` tensors): products and sums
 * rounded one at a time in k order, the bias added last (addmm's input
 * term).  style[r, n] = bf16(st[r, n]) (the table's bf16 cast);
 * fin[r, n - fin_col0] = st[r, n] for n >= fin_col0 (the final norm's
 * rows, kept fp32; fin NULL skips them).  w is bf16 [N, K] row-major (the
 * norms' dense weights concatenated along their outputs, norm i's chunks at
 * columns 3*D*i + {0, D, 2*D}); cond fp32 [rows, K]; bias fp32 [N] or NULL.
 * Reading: the weights are the modules' own bf16 values, which `.float()`
 * widens exactly.
 */
void or_style_project(int rows, int K, int N, const float *cond,
                      const uint16_t *w, const float *bias, uint16_t *style,
                      float *fin, int fin_col0)
{
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        const uint16_t *wr = w + (long)n * K;
        for (int r = 0; r < rows; ++r) {
            const float *cr = cond + (long)r * K;
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) acc = acc + cr[k] * or_bf16_to_f32(wr[k]);
            float st = bias ? acc + bias[n] : acc;
            style[(long)r * N + n] = or_bf16_from_f32(st);
            if (fin && n >= fin_col0) fin[(long)r * (N - fin_col0) + (n - fin_col0)] = st;
        }
    }
}

/* OpenMP thread count the oracle runs with (1 without OpenMP). */
int or_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
