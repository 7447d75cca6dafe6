// Host-side plan of one tensor-product convolution contract.
#pragma once

#include <string>
#include <vector>

#include "common.cuh"

namespace tpc {

struct Block {
  int mul, l, p, offset;
};

struct HostPath {
  int l1, p1, l2, p2, l3, p3;
  int i_in, i_out, mul_in, mul_out;
  int x_off, out_off;
  long long w_off, n_w;
  int nnz;
};

// Default bytes of one uvw state chunk (the scratch budget of Sobek App. B.2).
constexpr size_t kUvwChunkBytes = size_t(1) << 30;

struct Plan {
  int mode = 0;     // 0 uvu, 1 uvw
  bool per_path = false;    // uvu with one output block per path
  int schedule = 0;         // uvu forward: 0 streamed (Sobek §3.1), 1 receiver state (Sobek §4.2)
  int dtype = 0;    // 0 f32, 1 f64
  int K = 0, KP = 0, CPL = 1, sh_lmax = 0, lmax = 0;
  int fwd_CPL = 1;          // channels per lane of the forward kernel
  int edge_V = 1;           // channels per gather in the uvu backward edge pass
  int prof = 3;             // degree profile: 0 (2,2,2) 1 (1,3,3) 2 (3,3,3) 3 (4,4,4) 4 (6,6,6)
  int cy_stride = 0, fwd_chunk = 32, fwd_warp_smem = 0;
  int fwd_ring_off = 0, fwd_ring_g = 1;   // forward: x copy ring offset (bytes); group size (= fwd_ring_g())
  int src_cy_stride = 0, src_chunk = 32, src_warp_smem = 0;
  int src_ring_off = 0, src_ring_g = 1;   // source pass: m_bar ring offset (bytes); group size (= src_ring_g())
  bool src_split_ok = false;      // source pass: the split mode's x_bar partials fit beside the warps' slices
  std::vector<Block> bin, bout;
  std::vector<HostPath> paths;  // canonical enumeration order
  int c_in = 0, c_out = 0, dim_y = 0;
  long long n_w = 0;
  // kernel descriptor tables
  std::vector<TileD> out_tiles;   // (output block, channel tile), paths_by_out ranges
  std::vector<PathD> paths_by_out;
  std::vector<TileD> in_tiles;    // (input block, channel tile), paths_by_in ranges
  std::vector<PathD> paths_by_in;
  std::vector<int> in_tile_cost;  // source pass: estimated warp instructions per edge of each in_tiles entry
  std::vector<PathD> paths_canon;
  // second-order program: 32-channel tiles of the output and input blocks
  std::vector<TileD> dbl_out_tiles;
  std::vector<PathD> dbl_paths_by_out;
  std::vector<TileD> dbl_in_tiles;
  std::vector<int> dbl_in_tile_cost;   // per-edge cost estimate of each dbl_in_tiles entry
  std::vector<PathD> dbl_paths_by_in;
  bool dbl_ok = false;
  // fully connected (uvw) tables
  std::vector<UvwBlockD> uvw_out;   // output blocks, with paths_fwd ranges
  std::vector<PathD> paths_fwd;     // by output block; gathered = x block
  std::vector<UvwBlockD> uvw_in;    // input blocks, with paths_adj ranges
  std::vector<PathD> paths_adj;     // by input block; gathered = grad_out block
  UvwPackParams pack{};
  long long s_row_elems = 0;        // state elements per receiver (S)
  long long sa_row_elems = 0;       // state elements per source (S')
  bool uvw_tc = false;              // channel mixing on the tensor cores (fp32)
  size_t state_budget = kUvwChunkBytes;   // bytes of one uvw state chunk
};


// Parse spherical-harmonic irreps "1x0e+1x1o+..." (degrees 0..L in order,
// multiplicity 1) into L and the parity of each degree.
int parse_sh_irreps(const char* s, int& sh_lmax, std::vector<int>& parity, std::string& msg);

// Owners per uvw state chunk for a problem of n_nodes nodes (dir 0: S, 1: S').
int uvw_chunk_rows(const Plan& p, long long n_nodes, int dir);

// Returns 0 or a negative tp_status; msg receives a human-readable reason.
// sh_parity: parity (+1 / -1) of the spherical-harmonic block of each degree
// 0..sh_lmax, or NULL for the natural parity (-1)^l.
int make_plan(const char* irreps_in, int sh_lmax, const char* irreps_out, int n_radial, int mode,
              int dtype, Plan& out, std::string& msg, const int* sh_parity = nullptr);

// CTAs of the double-backward source pass (kDbWarps warps each, one source
// stream per warp), dealt to its 32-channel input tiles in proportion to their
// per-edge cost as the first-order pass does; cta as in uvu_src_partition.
// Returns the A_bar partial slots (the largest per-tile warp count).
int uvu_dbl_src_partition(const Plan& p, long long n_nodes, int* cta);

// CTAs of the first-order source pass, dealt to the input-block tiles in
// proportion to their per-edge cost (one wave; at least one CTA per tile, and
// no more warps per tile than sources): tile t gets CTAs [cta[t], cta[t + 1])
// when cta (n_tiles + 1 entries) is not null. Returns the A_bar partial slots,
// the largest per-tile warp count capped at max_slots (each warp owns one slot
// of its tile's columns and serves every slots-th source). On graphs with too
// few (source, tile) pairs to fill the GPU, *split (when not null) is set to
// the warps of a CTA, which then share each source and deal the tile's paths;
// a slot is then a CTA's. Otherwise *split = 1.
int uvu_src_partition(const Plan& p, long long n_nodes, long long max_slots, int* cta, int* split = nullptr);

// Bytes of workspace for pass 0 (forward) or 1 (backward) at n_nodes receivers.
size_t workspace_bytes(const Plan& p, long long n_nodes, int pass);

// Algorithmic flops and compulsory bytes of one pass (0 fwd, 1 bwd).
void work_model(const Plan& p, long long n_nodes, long long n_edges, int pass, double& flops,
                double& bytes);

}  // namespace tpc
