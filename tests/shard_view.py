"""The one-rank-per-GPU view of a single-buffer layout, by its definition:
rank d's receive rows are rows [rank_off[d], rank_off[d+1]) of the
single-buffer layout, shifted to start at 0; a slot's destination rank is
e / L. Test helper: used by the GPU tests and pinned on the CPU by
tests/golden/shard_example.txt."""
import numpy as np

import oracle


def shard_view(idx: np.ndarray, lay: dict, R: int, T: int, E: int) -> list[dict]:
    """Per rank s: dst_rank / dst_row of its own slots, its count row, and,
    as a destination, recv_count, recv_off and the source token of each of its
    receive rows."""
    L = E // R
    dst, eoff, roff = lay["dst_row"], lay["expert_off"], lay["rank_off"]
    valid = dst >= 0
    N, K = idx.shape
    src_of_row = np.repeat(np.arange(N), K).reshape(N, K)[valid][np.argsort(dst[valid])].astype(np.int32)
    out = []
    for s in range(R):
        rows = slice(s * T, (s + 1) * T)
        v = idx[rows] >= 0
        d_rank = np.where(v, idx[rows] // L, 0).astype(np.uint8)
        d_row = np.where(v, dst[rows] - roff[d_rank], -1).astype(np.int32)
        out.append(dict(
            dst_rank=d_rank, dst_row=d_row, cnt_row=lay["cnt"][s].copy(),
            local_rows=oracle.layout(np.ascontiguousarray(idx[rows]), 1, T, E)["dst_row"],
            recv_count=lay["num_tokens_per_expert"][s * L:(s + 1) * L].copy(),
            recv_off=(eoff[s * L:(s + 1) * L + 1] - eoff[s * L]).astype(np.int32),
            recv_src=src_of_row[roff[s]:roff[s + 1]]))
    return out
