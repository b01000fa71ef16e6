/* A plain C caller of the attention library, linked against libattn.so with
 * no Python in between. It makes host-side calls only (version, status text,
 * workspace sizing, and a call the library must refuse before any launch),
 * so it runs without a GPU. Prints one line of results for the test. */
#include <stdio.h>
#include <string.h>

#include "attn.h"

/* A contiguous [n0, n1, n2, n3] view over `data` (never dereferenced here). */
static attn_tensor view4(void* data, int32_t dtype, int64_t n0, int64_t n1, int64_t n2, int64_t n3) {
  attn_tensor t;
  memset(&t, 0, sizeof t);
  t.data = data;
  t.dtype = dtype;
  t.ndim = 4;
  t.shape[0] = n0;
  t.shape[1] = n1;
  t.shape[2] = n2;
  t.shape[3] = n3;
  t.stride[3] = 1;
  t.stride[2] = n3;
  t.stride[1] = n2 * n3;
  t.stride[0] = n1 * n2 * n3;
  return t;
}

int main(void) {
  if (attn_version() != ATTN_VERSION) {
    printf("version mismatch: library %d, header %d\n", attn_version(), ATTN_VERSION);
    return 1;
  }
  /* Causal GQA problem: B=1, Hq=4, Hkv=2, T=300, d=dv=128, bf16. */
  void* fake = (void*)0x100000;
  attn_tensor q = view4(fake, ATTN_BF16, 1, 4, 300, 128);
  attn_tensor k = view4(fake, ATTN_BF16, 1, 2, 300, 128);
  attn_tensor v = view4(fake, ATTN_BF16, 1, 2, 300, 128);
  attn_mask m;
  memset(&m, 0, sizeof m);
  m.flags = ATTN_MASK_CAUSAL;
  size_t fwd_ws = attn_fwd_workspace_size(&q, &k, &v, &m);
  size_t bwd_ws = attn_bwd_workspace_size(&q, &k, &v, &m);

  /* Three K/V heads cannot serve four query heads: refused on the host. */
  attn_tensor k3 = view4(fake, ATTN_BF16, 1, 3, 300, 128);
  attn_tensor v3 = view4(fake, ATTN_BF16, 1, 3, 300, 128);
  attn_tensor o = view4(fake, ATTN_BF16, 1, 4, 300, 128);
  attn_tensor lse = view4(fake, ATTN_F32, 1, 4, 300, 1);
  lse.ndim = 3;
  attn_status st = attn_fwd(&q, &k3, &v3, &m, 0.088f, &o, &lse, fake, (size_t)1 << 20, NULL);

  printf("fwd_ws %zu bwd_ws %zu status %d %s\n", fwd_ws, bwd_ws, (int)st, attn_status_string(st));
  return st == ATTN_ERR_INVALID_ARG ? 0 : 2;
}
