"""The allocation-free MoE permutation (bsg_moe_permute_noalloc), for callers that cannot allocate
device memory -- a plugin whose host application owns every allocation, a serving loop that must not
call cudaMalloc / cudaFree because they can synchronise the device, a process whose device footprint
is fixed after start-up.  Its scratch is a fixed array inside the library, so the test checks, through
the C ABI, that two calls in a row (the second one reusing the array the first one left behind) give
exactly what the workspace entry point gives on the same routing.  The file name makes pytest collect
it last; it passes alone in a fresh process too."""
import numpy as np
import pytest
import torch

import nvfp4_grouped_gemm_indices_b200 as bsg

pytestmark = pytest.mark.gpu


def routing(T, top_k, G, seed):
    rng = np.random.default_rng(seed)
    ranks = np.arange(1, G + 1, dtype=np.float64) ** -1.2
    p = ranks / ranks.sum()
    ids = rng.choice(G, size=(T, top_k), p=p[rng.permutation(G)]).astype(np.int32)
    ids[rng.random((T, top_k)) < 0.02] = -1                     # a few dropped entries
    return torch.from_numpy(ids).cuda()


def outputs(T, top_k, G):
    n = T * top_k
    return [torch.full((n,), 0x5EED, dtype=torch.int32, device="cuda"),
            torch.full((n,), 0x5EED, dtype=torch.int32, device="cuda"),
            torch.full((T, top_k), 0x5EED, dtype=torch.int32, device="cuda"),
            torch.full((G + 1,), 0x5EED, dtype=torch.int32, device="cuda")]


@pytest.mark.parametrize("T,top_k,G", [(8192, 8, 64), (512, 8, 64)])
def test_noalloc_permute_matches_the_workspace_entry_point_twice_in_a_row(T, top_k, G):
    # 65536 entries take the three-launch path through the static scratch (64 KiB of counters);
    # 4096 take the single-CTA path, which needs no scratch
    need = bsg.bsg_moe_permute_workspace_size(T, top_k, G)
    assert need == (65536 if T == 8192 else 0)
    ws = torch.empty(max(16, need), dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((1, 2)):                         # two calls in a row
        ids = routing(T, top_k, G, seed)
        ref = outputs(T, top_k, G)
        bsg.bsg_moe_permute(ids, T, top_k, G, *ref, ws, ws.numel())
        got = outputs(T, top_k, G)
        bsg.bsg_moe_permute_noalloc(ids, T, top_k, G, *got)
        torch.cuda.synchronize()
        for name, a, b in zip(("src_rows", "m_indices", "dst_rows", "expert_offsets"), got, ref):
            assert torch.equal(a, b), f"call {call}: {name} differs"


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    T, top_k, G = 1 << 16, 8, 4096                              # needs 8 MiB of counters
    ids = torch.zeros((1, 1), dtype=torch.int32, device="cuda")  # never read: the call launches nothing
    out = outputs(1, 1, 1)
    with pytest.raises(bsg.BsgError) as ei:
        bsg.bsg_moe_permute_noalloc(ids, T, top_k, G, *out)
    assert ei.value.status == bsg.BSG_ERR_UNSUPPORTED_SHAPE and "2097152 bytes" in str(ei.value)
