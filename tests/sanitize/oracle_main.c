/* Drives every oracle function once on small shapes so the oracle can be
 * built and run under AddressSanitizer and UndefinedBehaviorSanitizer
 * (tests/test_oracle_sanitizers.py).  The inputs are arbitrary; only memory
 * and arithmetic errors are looked for here. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

int orc_route(int, int, int, int, const float*, const float*, int32_t*, float*);
int orc_route_limited(int, int, int, int, int, int, const float*, const float*, int32_t*, float*);
void orc_bias_update(int, int64_t, const int32_t*, float, const float*, float*);
int64_t orc_layout_rows(int, int, int, int, int);
int orc_layout(int, int, int, int, int, int, const int32_t*, int32_t*, int32_t*, int32_t*,
               int32_t*, int32_t*, int32_t*);
int64_t orc_layout_src_rows(int, int, int, int, int, int);
int orc_layout_src(int, int, int, int, int, int, const int32_t*, int32_t*, int32_t*, int32_t*,
                   int32_t*, int32_t*, int32_t*, int32_t*);
int orc_layout_remote_first(int, int, int, int, int, int, int, const int32_t*, int32_t*,
                            int32_t*, int32_t*, int32_t*, int32_t*, int32_t*, int32_t*);
void orc_route_round_robin(int, int, int, int32_t*, float*);
void orc_dispatch_bf16(int, int, int, const uint16_t*, const int32_t*, uint16_t*);
void orc_dispatch_fp8(int, int, int, const uint16_t*, const int32_t*, uint8_t*, float*);
void orc_combine(int, int, int, const uint16_t*, const int32_t*, const float*, const uint16_t*,
                 const uint16_t*, uint16_t*, const int32_t*, int);
void orc_combine_f32(int, int, int, const uint16_t*, const int32_t*, const float*, const uint16_t*,
                 const uint16_t*, uint16_t*, const int32_t*, int);
void orc_dequant_fp8(int64_t, int, const uint8_t*, const float*, uint16_t*);
uint8_t orc_e4m3_encode_satfinite(float);
double orc_e4m3_decode(uint8_t);
uint16_t orc_double_to_bf16(double);

static void* xmalloc(size_t n) {
  void* p = malloc(n ? n : 1);
  if (!p) exit(2);
  return p;
}

static int run(int T, int E, int k, int R, int C, int align, int H) {
  float* logits = xmalloc(sizeof(float) * T * E);
  float* bias = xmalloc(sizeof(float) * E);
  for (int i = 0; i < T * E; ++i) logits[i] = (float)((i * 7919) % 1000) / 250.0f - 2.0f;
  for (int e = 0; e < E; ++e) bias[e] = (float)(e % 5) * 0.01f;
  int32_t* ids = xmalloc(sizeof(int32_t) * T * k);
  float* gates = xmalloc(sizeof(float) * T * k);
  if (orc_route(T, E, k, 1, logits, bias, ids, gates)) return 1;
  if (orc_route(T, E, k, 0, logits, NULL, ids, gates)) return 1;
  if (R > 1 && orc_route_limited(T, E, k, R, R - 1, 1, logits, bias, ids, gates)) return 1;
  orc_route_round_robin(T, E, k, ids, gates);
  if (orc_route(T, E, k, 1, logits, bias, ids, gates)) return 1;

  const int64_t N = orc_layout_rows(T, E, k, C, align);
  int32_t *counts = xmalloc(4 * E), *eoff = xmalloc(4 * (E + 1)), *roff = xmalloc(4 * (R + 1));
  int32_t *rc = xmalloc(4 * R), *dst = xmalloc(4 * T * k), *src = xmalloc(4 * (N ? N : 1));
  if (orc_layout(T, E, k, R, C, align, ids, counts, eoff, roff, rc, dst, src)) return 1;
  int32_t* tiles = xmalloc(4 * (N / align + 1));
  if (orc_layout_remote_first(T, E, k, R, C, align, R / 2, ids, counts, eoff, roff, rc, dst, src,
                              tiles))
    return 1;
  float* b2 = xmalloc(sizeof(float) * E);
  orc_bias_update(E, (int64_t)T * k, counts, 0.01f, bias, b2);

  const int64_t Ns = orc_layout_src_rows(T, E, k, R, C, align);
  int32_t *sc = xmalloc(4 * R * E), *so = xmalloc(4 * (R * E + 1)), *pc = xmalloc(4 * R * R);
  int32_t *dst2 = xmalloc(4 * T * k), *src2 = xmalloc(4 * (Ns ? Ns : 1));
  if (orc_layout_src(T, E, k, R, C, align, ids, sc, so, pc, roff, rc, dst2, src2)) return 1;

  if (orc_layout(T, E, k, R, C, align, ids, counts, eoff, roff, rc, dst, src)) return 1;
  uint16_t* x = xmalloc(2 * T * H);
  for (int i = 0; i < T * H; ++i) x[i] = orc_double_to_bf16((double)((i * 31) % 97) / 13.0 - 3.0);
  uint16_t* xd = xmalloc(2 * (N ? N : 1) * H);
  orc_dispatch_bf16(T, H, k, x, dst, xd);
  uint16_t* out = xmalloc(2 * T * H);
  int32_t tok[2] = {0, T - 1};
  orc_combine(T, H, k, xd, dst, gates, x, x, out, NULL, 0);
  orc_combine(T, H, k, xd, dst, gates, NULL, NULL, out, tok, T > 0 ? 2 : 0);
  orc_combine_f32(T, H, k, xd, dst, gates, x, x, out, NULL, 0);
  orc_combine_f32(T, H, k, xd, dst, gates, NULL, NULL, out, tok, T > 0 ? 2 : 0);
  if (H % 128 == 0) {
    uint8_t* q = xmalloc((N ? N : 1) * H);
    float* s = xmalloc(4 * (N ? N : 1) * (H / 128));
    orc_dispatch_fp8(T, H, k, x, dst, q, s);
    orc_dequant_fp8(N, H, q, s, xd);
    free(q);
    free(s);
  }
  free(logits); free(bias); free(ids); free(gates); free(counts); free(eoff); free(roff);
  free(rc); free(dst); free(src); free(tiles); free(b2); free(sc); free(so); free(pc);
  free(dst2); free(src2); free(x); free(xd); free(out);
  return 0;
}

int main(void) {
  for (int c = 0; c < 256; ++c) (void)orc_e4m3_decode((uint8_t)c);
  for (int i = -2000; i <= 2000; ++i) (void)orc_e4m3_encode_satfinite((float)i * 0.37f);
  int bad = 0;
  bad |= run(37, 16, 3, 4, 0, 1, 128);
  bad |= run(37, 16, 3, 4, 0, 8, 64);
  bad |= run(50, 12, 4, 3, 5, 1, 256);
  bad |= run(3, 8, 2, 4, 0, 4, 16);
  bad |= run(1, 1, 1, 1, 0, 1, 8);
  bad |= run(0, 8, 2, 2, 2, 1, 128);
  bad |= run(120, 256, 8, 32, 0, 1, 128);
  printf(bad ? "oracle run failed\n" : "oracle sanitizer run ok\n");
  return bad;
}
