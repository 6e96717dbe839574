// Tensor-map (TMA descriptor) encoding through the driver entry point.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include <string>

// Resolve cuTensorMapEncodeTiled once; false (with a message) if unavailable.
bool tmap_init(std::string& err);

// bf16 matrix [rows, cols] row-major with row stride ld elements; box
// (64 columns, box_rows rows), 128-byte swizzle; out-of-range reads are zero.
bool tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
                  std::string& err);

// 8-bit matrix (e4m3 codes) [rows, cols] row-major with row stride ld bytes
// (a multiple of 16); box (128 columns = 128 bytes, box_rows rows), 128-byte
// swizzle; out-of-range reads are zero.
bool tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
                std::string& err);

// bf16 stack of [H, rows, d] planes: dims (d, rows, H, slices), dense; box
// (64, 128, 1, 1), 128-byte swizzle; rows beyond `rows` read as zero.
bool tmap_planes_bf16(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows, uint64_t H, uint64_t slices,
                     std::string& err);
// 8-bit (e4m3 codes) stack of [H, rows, d] planes, d = 128: dims (d, rows, H,
// slices), dense; box (128, 128, 1, 1), 128-byte swizzle; rows beyond `rows`
// read as zero.
bool tmap_planes_u8(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows, uint64_t H, uint64_t slices,
                    std::string& err);
