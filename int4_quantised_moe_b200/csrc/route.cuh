#pragma once
#include "common.cuh"

namespace r4 {

constexpr int kRouteChunk = 1024;  // flat slots per block of the counting sort
constexpr int kTileRows = 192;     // max permuted rows (tokens) per GEMM tile (a TMEM accumulator's columns)
// max rows per tile in the narrow GEMM configuration (layers with few rows per expert)
constexpr int kTileRowsNarrow = 64;

size_t route_scratch_bytes(int32_t routed_slots, int32_t experts);

// ids int64 [qlen, top_k]; rw fp32 [qlen, top_k] (may be null when w_perm is null)
// Writes offsets [E+1], perm [routed], inv [qlen*top_k], w_perm [routed] (optional),
// tok_tiles (int4 {expert, first row, rows, 0}) and hdr->{routed, n_tok_tiles, qlen}.
// tile_rows (a multiple of 16): the most rows of a tile; an expert's rows are
// cut into ceil(rows / tile_rows) tiles of equal size rounded up to 16.
cudaError_t launch_route(const int64_t* ids, const float* rw, int32_t qlen, int32_t top_k, int32_t experts,
                         int32_t* offsets, int32_t* perm, int32_t* inv, float* w_perm, int4* tok_tiles,
                         int32_t* block_hist, WsHeader* hdr, cudaStream_t stream, int32_t tile_rows = kTileRows);

__global__ void tail_fill_kernel(int32_t* perm, const int32_t* offsets, int32_t experts, int32_t total);

inline int32_t max_tok_tiles(int32_t routed_slots, int32_t experts, int32_t tile_rows = kTileRows) {
  // every expert's rows split into ceil(n/tile_rows) tiles: at most E + slots/tile_rows tiles
  return experts + (routed_slots + tile_rows - 1) / tile_rows;
}

}  // namespace r4
