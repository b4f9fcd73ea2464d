/* A plain C99 caller of the FLCE C ABI: no C++, no PyTorch, only the CUDA
 * runtime for device memory and a stream.
 *
 *   flce_c_driver IN OUT
 *
 * IN holds a header (struct in_header below) followed by hidden [N*H] and
 * weight [V*H] as bf16 bit patterns and labels [N] as int64.  The driver runs
 * flce_forward and flce_backward (bf16 path, grad_output = 1, the library's
 * own count) on one stream, reads the workspace status, and writes to OUT a
 * header (struct out_header) followed by lse [N], d_hidden [N*H] and
 * d_weight [V*H] as float32.  Exit status 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "flce.h"

struct in_header {
  char magic[8]; /* "FLCEIN1" */
  int64_t N, H, V, ignore_index;
  float softcap, grad_scale;
  int32_t reduction, reserved;
};

struct out_header {
  char magic[8]; /* "FLCEOUT" */
  float loss;
  uint32_t status;
  int64_t num_tokens;
};

#define CK(x)                                                                  \
  do {                                                                         \
    cudaError_t e_ = (x);                                                      \
    if (e_ != cudaSuccess) {                                                   \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));                 \
      return 2;                                                                \
    }                                                                          \
  } while (0)

#define FL(x)                                                                  \
  do {                                                                         \
    flce_status s_ = (x);                                                      \
    if (s_ != FLCE_OK) {                                                       \
      fprintf(stderr, "%s: %s\n", #x, flce_status_string(s_));                 \
      return 3;                                                                \
    }                                                                          \
  } while (0)

static void* read_block(FILE* f, size_t bytes) {
  void* p = malloc(bytes ? bytes : 1);
  if (p != NULL && bytes && fread(p, 1, bytes, f) != bytes) {
    free(p);
    return NULL;
  }
  return p;
}

int main(int argc, char** argv) {
  struct in_header hin;
  struct out_header hout;
  FILE* fin;
  FILE* fout;
  size_t nh, vh, wsb;
  void *h_hid, *h_w, *h_y, *d_hid, *d_w, *d_ws;
  int64_t *d_y, *d_ntok;
  float *d_loss, *d_lse, *d_dh, *d_dw, *h_lse, *h_dh, *h_dw;
  cudaStream_t st;

  if (argc != 3) {
    fprintf(stderr, "usage: %s IN OUT\n", argv[0]);
    return 1;
  }
  fin = fopen(argv[1], "rb");
  if (fin == NULL || fread(&hin, sizeof hin, 1, fin) != 1 || memcmp(hin.magic, "FLCEIN1", 8)) {
    fprintf(stderr, "bad input file\n");
    return 1;
  }
  nh = (size_t)hin.N * (size_t)hin.H;
  vh = (size_t)hin.V * (size_t)hin.H;
  h_hid = read_block(fin, 2 * nh);
  h_w = read_block(fin, 2 * vh);
  h_y = read_block(fin, 8 * (size_t)hin.N);
  fclose(fin);
  if (h_hid == NULL || h_w == NULL || h_y == NULL) {
    fprintf(stderr, "short input file\n");
    return 1;
  }

  wsb = flce_workspace_bytes(hin.N, hin.H, hin.V, FLCE_BF16);
  if (wsb == 0) {
    fprintf(stderr, "invalid sizes\n");
    return 1;
  }
  CK(cudaStreamCreate(&st));
  CK(cudaMalloc(&d_hid, 2 * nh));
  CK(cudaMalloc(&d_w, 2 * vh));
  CK(cudaMalloc((void**)&d_y, 8 * (size_t)hin.N));
  CK(cudaMalloc((void**)&d_loss, sizeof(float)));
  CK(cudaMalloc((void**)&d_ntok, sizeof(int64_t)));
  CK(cudaMalloc((void**)&d_lse, 4 * (size_t)hin.N));
  CK(cudaMalloc((void**)&d_dh, 4 * nh));
  CK(cudaMalloc((void**)&d_dw, 4 * vh));
  CK(cudaMalloc(&d_ws, wsb));
  CK(cudaMemcpyAsync(d_hid, h_hid, 2 * nh, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(d_w, h_w, 2 * vh, cudaMemcpyHostToDevice, st));
  CK(cudaMemcpyAsync(d_y, h_y, 8 * (size_t)hin.N, cudaMemcpyHostToDevice, st));

  FL(flce_forward(d_hid, d_w, d_y, hin.N, hin.H, hin.V, hin.ignore_index, hin.softcap,
                  hin.reduction, FLCE_BF16, d_loss, d_ntok, d_lse, d_ws, wsb, st));
  memset(&hout, 0, sizeof hout);
  hout.status = (uint32_t)flce_get_status(d_ws, st); /* the forward's device-side errors */
  FL(flce_backward(d_hid, d_w, d_y, d_lse, hin.N, hin.H, hin.V, hin.ignore_index, hin.softcap,
                   hin.reduction, FLCE_BF16, NULL, hin.grad_scale, NULL, d_dh, d_dw, 0, d_ws,
                   wsb, st));
  hout.status |= (uint32_t)flce_get_status(d_ws, st) << 8; /* and the backward's */

  h_lse = (float*)malloc(4 * (size_t)hin.N);
  h_dh = (float*)malloc(4 * nh);
  h_dw = (float*)malloc(4 * vh);
  if (h_lse == NULL || h_dh == NULL || h_dw == NULL) return 1;
  memcpy(hout.magic, "FLCEOUT", 8);
  CK(cudaMemcpy(&hout.loss, d_loss, sizeof(float), cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&hout.num_tokens, d_ntok, sizeof(int64_t), cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(h_lse, d_lse, 4 * (size_t)hin.N, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(h_dh, d_dh, 4 * nh, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(h_dw, d_dw, 4 * vh, cudaMemcpyDeviceToHost));

  fout = fopen(argv[2], "wb");
  if (fout == NULL || fwrite(&hout, sizeof hout, 1, fout) != 1 ||
      fwrite(h_lse, 4, (size_t)hin.N, fout) != (size_t)hin.N || fwrite(h_dh, 4, nh, fout) != nh ||
      fwrite(h_dw, 4, vh, fout) != vh) {
    fprintf(stderr, "cannot write output\n");
    return 1;
  }
  fclose(fout);
  cudaFree(d_hid);
  cudaFree(d_w);
  cudaFree(d_y);
  cudaFree(d_loss);
  cudaFree(d_ntok);
  cudaFree(d_lse);
  cudaFree(d_dh);
  cudaFree(d_dw);
  cudaFree(d_ws);
  cudaStreamDestroy(st);
  free(h_hid);
  free(h_w);
  free(h_y);
  free(h_lse);
  free(h_dh);
  free(h_dw);
  return 0;
}
