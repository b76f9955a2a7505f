/* A plain C99 client of libmoe: the boundary used without Python or C++.
 *
 *   moe_c_client validate
 *       host-only calls: sizes, capacities, status strings and argument validation (no GPU needed;
 *       every call here returns before launching anything)
 *   moe_c_client forward <in.bin> <out.bin>
 *       one fp32 layer forward on the GPU through moe_forward.  in.bin: int32 T, H, E, k, F, then
 *       fp32 x[T,H] Wg[H,E] bg[E] W1[E,H,F] b1[E,F] W2[E,F,H] b2[E,H] (dropless, GELU).  out.bin:
 *       fp32 out[T,H], int32 topk_idx[T,k], fp32 aux_loss, z_loss.
 * Exit status 0 on success; a message on stderr otherwise. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "moe.h"

#define CHECK(cond, msg)                                  \
  do {                                                    \
    if (!(cond)) {                                        \
      fprintf(stderr, "moe_c_client: %s\n", msg);         \
      return 1;                                           \
    }                                                     \
  } while (0)

static moe_shape_t make_shape(int T, int H, int E, int k, int F, double cf, moe_dtype_t dt) {
  moe_shape_t s;
  memset(&s, 0, sizeof s); /* zero-initialised: GELU, token choice, no min_capacity */
  s.T = T;
  s.H = H;
  s.E = E;
  s.k = k;
  s.F = F;
  s.capacity_factor = cf;
  s.dtype = dt;
  return s;
}

static int validate(void) {
  moe_shape_t s = make_shape(8192, 1024, 128, 1, 4096, 1.25, MOE_DTYPE_BF16);
  CHECK(moe_capacity(&s) == 80, "capacity of the Switch-shaped layer is not 80");
  CHECK(moe_workspace_size(&s) > 0, "workspace size of a valid shape is 0");
  s.capacity_factor = INFINITY;
  CHECK(moe_capacity(&s) == -1, "dropless capacity is not -1");
  moe_shape_t bad = make_shape(64, 64, 4, 5, 64, INFINITY, MOE_DTYPE_F32); /* k > E */
  CHECK(moe_workspace_size(&bad) == 0, "invalid shape has a workspace size");
  CHECK(moe_capacity(&bad) == -2, "invalid shape has a capacity");
  moe_io_t io;
  memset(&io, 0, sizeof io);
  CHECK(moe_forward(&bad, &io, NULL, 0, 0) == MOE_ERR_INVALID_ARG, "invalid shape accepted by moe_forward");
  moe_shape_t ok = make_shape(64, 64, 4, 2, 64, INFINITY, MOE_DTYPE_F32);
  CHECK(moe_forward(&ok, &io, NULL, 0, 0) == MOE_ERR_INVALID_ARG, "null io pointers accepted");
  CHECK(moe_forward(&ok, NULL, NULL, 0, 0) == MOE_ERR_INVALID_ARG, "null io accepted");
  CHECK(moe_losses_from_sums(0, NULL, NULL, NULL, 0) == MOE_ERR_INVALID_ARG, "E = 0 accepted");
  CHECK(strlen(moe_status_string(MOE_ERR_WORKSPACE)) > 0, "empty status string");
  printf("validate ok\n");
  return 0;
}

static int read_all(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n; }

static int forward(const char* in_path, const char* out_path) {
  FILE* f = fopen(in_path, "rb");
  CHECK(f != NULL, "cannot open the input file");
  int32_t dims[5];
  CHECK(read_all(f, dims, sizeof dims), "short input file");
  const int T = dims[0], H = dims[1], E = dims[2], k = dims[3], F = dims[4];
  const size_t n[7] = {(size_t)T * H, (size_t)H * E, (size_t)E, (size_t)E * H * F, (size_t)E * F,
                       (size_t)E * F * H, (size_t)E * H};
  float* host[7];
  void* dev[7];
  for (int i = 0; i < 7; ++i) {
    host[i] = (float*)malloc(n[i] * sizeof(float));
    CHECK(host[i] != NULL, "out of host memory");
    CHECK(read_all(f, host[i], n[i] * sizeof(float)), "short input file");
    CHECK(cudaMalloc(&dev[i], n[i] * sizeof(float)) == cudaSuccess, "cudaMalloc failed");
    CHECK(cudaMemcpy(dev[i], host[i], n[i] * sizeof(float), cudaMemcpyHostToDevice) == cudaSuccess,
          "copy to the device failed");
  }
  fclose(f);

  moe_shape_t s = make_shape(T, H, E, k, F, INFINITY, MOE_DTYPE_F32);
  const size_t ws_bytes = moe_workspace_size(&s);
  CHECK(ws_bytes > 0, "invalid shape");
  void *ws, *out, *idx, *w, *counts, *dropped, *losses;
  CHECK(cudaMalloc(&ws, ws_bytes) == cudaSuccess, "cudaMalloc(ws) failed");
  CHECK(cudaMemset(ws, 0, 256) == cudaSuccess, "clearing the error word failed");
  CHECK(cudaMalloc(&out, (size_t)T * H * sizeof(float)) == cudaSuccess, "cudaMalloc(out) failed");
  CHECK(cudaMalloc(&idx, (size_t)T * k * sizeof(int32_t)) == cudaSuccess, "cudaMalloc(idx) failed");
  CHECK(cudaMalloc(&w, (size_t)T * k * sizeof(float)) == cudaSuccess, "cudaMalloc(w) failed");
  CHECK(cudaMalloc(&counts, (size_t)E * sizeof(int32_t)) == cudaSuccess, "cudaMalloc(counts) failed");
  CHECK(cudaMalloc(&dropped, (size_t)T * k) == cudaSuccess, "cudaMalloc(dropped) failed");
  CHECK(cudaMalloc(&losses, 2 * sizeof(float)) == cudaSuccess, "cudaMalloc(losses) failed");

  moe_io_t io;
  io.x = dev[0];
  io.Wg = dev[1];
  io.bg = dev[2];
  io.W1 = dev[3];
  io.b1 = dev[4];
  io.W2 = dev[5];
  io.b2 = dev[6];
  io.out = (float*)out;
  io.topk_idx = (int32_t*)idx;
  io.topk_w = (float*)w;
  io.expert_counts = (int32_t*)counts;
  io.dropped = (uint8_t*)dropped;
  io.aux_loss = (float*)losses;
  io.z_loss = (float*)losses + 1;
  CHECK(moe_forward(&s, &io, ws, ws_bytes, 0) == MOE_OK, "moe_forward refused the call");
  CHECK(moe_get_device_status(ws, 0) == MOE_OK, "device status is not OK");

  float* hout = (float*)malloc((size_t)T * H * sizeof(float));
  int32_t* hidx = (int32_t*)malloc((size_t)T * k * sizeof(int32_t));
  float hl[2];
  CHECK(hout != NULL && hidx != NULL, "out of host memory");
  CHECK(cudaMemcpy(hout, out, (size_t)T * H * sizeof(float), cudaMemcpyDeviceToHost) == cudaSuccess, "copy back");
  CHECK(cudaMemcpy(hidx, idx, (size_t)T * k * sizeof(int32_t), cudaMemcpyDeviceToHost) == cudaSuccess, "copy back");
  CHECK(cudaMemcpy(hl, losses, sizeof hl, cudaMemcpyDeviceToHost) == cudaSuccess, "copy back");
  FILE* o = fopen(out_path, "wb");
  CHECK(o != NULL, "cannot open the output file");
  CHECK(fwrite(hout, sizeof(float), (size_t)T * H, o) == (size_t)T * H, "short write");
  CHECK(fwrite(hidx, sizeof(int32_t), (size_t)T * k, o) == (size_t)T * k, "short write");
  CHECK(fwrite(hl, sizeof(float), 2, o) == 2, "short write");
  fclose(o);
  printf("forward ok\n");
  return 0;
}

int main(int argc, char** argv) {
  if (argc >= 2 && strcmp(argv[1], "validate") == 0) return validate();
  if (argc >= 4 && strcmp(argv[1], "forward") == 0) return forward(argv[2], argv[3]);
  fprintf(stderr, "usage: moe_c_client validate | forward <in.bin> <out.bin>\n");
  return 2;
}
