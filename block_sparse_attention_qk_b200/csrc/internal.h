// Launcher interface between the C ABI layer (api.cu) and the kernels.
#pragma once

#include "common.cuh"

namespace sbattn {

// Host-side argument checks shared by the entry points (api.cu).
bool aligned16(const void* p);
int nblk_of(long long N);
int check_dims(long long B, long long N, long long H, long long d);
int check_select_outputs(const int32_t* kept_idx, const int32_t* kept_cnt, const float* scores);

struct PrologueArgs {
  const uint16_t* q;   // input rows (prologue: raw Q; pooling: rotated Q)
  const uint16_t* k;
  const uint16_t* w_q;
  const uint16_t* w_k;
  uint16_t* q_out;
  uint16_t* k_out;
  float* q_pool;       // [B, H, nblk, d] or null
  float* k_pool;
  int B, N, H, T, Hh, W, nblk;
  int dim_t, dim_h, dim_w;
  float theta, eps;
};

// Largest rotation table the prologue keeps in shared memory.
constexpr size_t kMaxRopeTableBytes = 160 * 1024;
size_t prologue_table_bytes(int T, int Hh, int W, int dim_t, int dim_h, int dim_w);
int launch_prologue(const PrologueArgs& a, cudaStream_t stream);
int launch_pool(const PrologueArgs& a, cudaStream_t stream);

struct DitArgs {  // AdaLN modulation
  const uint16_t* x;      // [B, N, C]
  const uint16_t* shift;  // [B, C]
  const uint16_t* scale;  // [B, C]
  uint16_t* out;          // [B, N, C]
  int B, N, C;
  float eps;
};
constexpr int kMaxAdaLNChannels = 6144;
int launch_adaln(const DitArgs& a, cudaStream_t stream);

struct SwigluArgs {
  const uint16_t* gate;  // row r at gate + r * ld_in
  const uint16_t* up;
  uint16_t* out;         // [rows, F]
  long rows, ld_in;
  int F;
};
int launch_swiglu(const SwigluArgs& a, cudaStream_t stream);

struct SelectArgs {
  const float* q_bar;  // [B, H, nblk, d]
  const float* k_bar;
  int B, H, nblk;
  int keep;            // budget form: kept blocks per row (diagonal included)
  int threshold_mode;  // 1: keep score >= tau instead of a budget
  float tau;
  int32_t* kept_idx;   // [B, H, nblk, K_capacity]
  int32_t* kept_cnt;   // [B, H, nblk]
  int K_capacity;
  float* scores;       // [B, H, nblk, nblk] or null
};

// Largest nblk the selection kernel handles (one score row in shared memory).
int select_max_nblk();
int launch_select(const SelectArgs& a, cudaStream_t stream);

struct AttentionArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* kept_idx;
  const int32_t* kept_cnt;
  uint16_t* out;
  int32_t* status;
  int B, N, H, nblk, K_capacity;
  float scale;
  unsigned long long wait_limit_ns;  // limit of every bounded wait inside the kernel
  int withhold_v_tile;               // diagnostic: per-CTA V tile never copied (-1: none)
};

int launch_attention(const AttentionArgs& a, cudaStream_t stream);

// TMA descriptor of a [B, N, H, 128] bf16 tensor (box: 64 channels x 64 tokens
// of one head, 128-byte swizzle, zero fill past N).
int make_bf16_row_map(CUtensorMap* map, const void* base, int B, int N, int H);

}  // namespace sbattn
