// shared_prefix_plan.cu -- host planner for prefix-deduplicated decode when
// the sharing forms a tree (forks of forks: a common system prompt, then
// per-task prompts, then per-sample continuations).
//
// pa_shared_prefix_plan groups the sequences that start with the same
// physical block at the run of blocks ALL of them share, so blocks that only
// a sub-group shares are still read once per sequence.  Here the groups are
// chosen on the trie of the sequences' block paths instead.  A sequence's
// path is its table up to the block before the one holding its last token
// (those blocks are whole and leave it a token of its own).  A group formed
// at a trie node of depth d with k members saves (k - 1) * d block reads.
// Bottom-up, the sequences left ungrouped below a node are grouped there if
// that saves at least as much as the most the parent level could save for
// them, (k - 1) * d >= k * d_parent; otherwise they are passed up.  Every
// group formed below the common run saves at least its members' share of
// it, so the plan never saves less than the one-level one.
#include <algorithm>
#include <cstdint>
#include <numeric>
#include <utility>
#include <vector>

#include "paged_attention.h"
#include "pa_internal.h"

namespace {

struct Node {
  int depth;               // shared blocks of every sequence below
  std::vector<int> free;   // sequences below not grouped yet (sorted positions)
};

}  // namespace

extern "C" pa_status pa_shared_prefix_plan_tree(const int32_t* block_tables,
                                                const int32_t* context_lens, int num_seqs,
                                                int max_blocks_per_seq, int block_size,
                                                int min_shared_blocks, int32_t* group_seqs,
                                                int32_t* group_start, int32_t* group_blocks,
                                                int* num_groups, int* num_listed) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || !num_groups || !num_listed)
    return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
  *num_groups = 0;
  *num_listed = 0;
  if (num_seqs == 0) return PA_OK;
  if (!block_tables || !context_lens || !group_seqs || !group_start || !group_blocks)
    return PA_ERR_INVALID_ARG;
  const int min_blocks = min_shared_blocks > 1 ? min_shared_blocks : 1;
  const long long cap_len = static_cast<long long>(max_blocks_per_seq) * pa::kBlockSize;
  auto row = [&](int s) { return block_tables + static_cast<size_t>(s) * max_blocks_per_seq; };

  // eligible sequences and the length of their paths
  std::vector<int> seqs, len(num_seqs, 0);
  for (int s = 0; s < num_seqs; ++s) {
    const int n = context_lens[s];
    if (n <= 0 || n > cap_len) continue;
    len[s] = (n - 1) / pa::kBlockSize;
    if (len[s] >= min_blocks) seqs.push_back(s);
  }
  // paths in lexicographic order (a path before its extensions; equal paths
  // by sequence index), and the common prefix of neighbours
  std::sort(seqs.begin(), seqs.end(), [&](int a, int b) {
    const int m = std::min(len[a], len[b]);
    const int32_t *ra = row(a), *rb = row(b);
    for (int j = 0; j < m; ++j)
      if (ra[j] != rb[j]) return ra[j] < rb[j];
    return len[a] != len[b] ? len[a] < len[b] : a < b;
  });
  const int m = static_cast<int>(seqs.size());
  auto lcp = [&](int a, int b) {
    const int lim = std::min(len[a], len[b]);
    const int32_t *ra = row(a), *rb = row(b);
    int j = 0;
    while (j < lim && ra[j] == rb[j]) ++j;
    return j;
  };

  std::vector<std::pair<std::vector<int>, int>> groups;  // (members, shared blocks)
  // a node's ungrouped sequences: grouped here, or handed to the parent
  auto resolve = [&](Node& v, int parent_depth) -> std::vector<int> {
    const long long k = static_cast<long long>(v.free.size());
    if (k >= 2 && v.depth >= min_blocks && (k - 1) * v.depth >= k * parent_depth) {
      groups.emplace_back(std::move(v.free), v.depth);
      return {};
    }
    return std::move(v.free);
  };
  auto append = [](std::vector<int>& to, std::vector<int>&& from) {
    to.insert(to.end(), from.begin(), from.end());
  };

  std::vector<Node> stack;
  stack.push_back(Node{0, {}});  // root: different first blocks never share
  for (int i = 0; i <= m; ++i) {
    // i == m closes every open node
    const int l = i == 0 ? 0 : i == m ? 0 : lcp(seqs[i - 1], seqs[i]);
    while (stack.back().depth > l) {
      Node v = std::move(stack.back());
      stack.pop_back();
      // its parent: the node below it on the stack, or a new one at depth l
      const int parent_depth = std::max(stack.back().depth, l);
      std::vector<int> up = resolve(v, parent_depth);
      if (stack.back().depth >= l) {
        append(stack.back().free, std::move(up));
      } else {
        stack.push_back(Node{l, std::move(up)});
      }
    }
    if (i == m) break;
    const int s = seqs[i];
    if (stack.back().depth < l) stack.push_back(Node{l, {}});
    if (len[s] > stack.back().depth) {
      stack.push_back(Node{len[s], {s}});
    } else {
      stack.back().free.push_back(s);  // its path ends at this node
    }
  }

  for (auto& g : groups) std::sort(g.first.begin(), g.first.end());
  std::sort(groups.begin(), groups.end(),
            [](const auto& a, const auto& b) { return a.first[0] < b.first[0]; });
  int listed = 0;
  group_start[0] = 0;
  for (size_t g = 0; g < groups.size(); ++g) {
    for (int s : groups[g].first) group_seqs[listed++] = s;
    group_start[g + 1] = listed;
    group_blocks[g] = groups[g].second;
  }
  *num_groups = static_cast<int>(groups.size());
  *num_listed = listed;
  return PA_OK;
}
