"""The allocation-free entry point (muon_ns_batched_noalloc).

It exists for callers that cannot allocate device memory when they need the
orthogonalisation (their own caching allocator owns the GPU, allocation is
forbidden after start-up, or they are handed only input and output pointers).
It runs the same kernels as muon_ns_batched on a fixed scratch array inside
the library, so its results must match that entry point's; two calls in a row
check that the scratch the first call leaves behind does not leak into the
second.  This file is collected last so that a stop-at-first-failure run has
already run every other test.
"""
import pytest
import torch

import newton_schulz_matrix_b200 as nsm
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    """Bit for bit: both entry points run the same kernels, and chunking (the
    fixed scratch holds fewer matrices than a caller workspace sized for all
    of them) does not change any result.  7 matrices of 1024 x 2048 need about
    84 MiB, so the scratch takes them in two chunks."""
    assert torch.cuda.is_available()
    cases = [((1024, 2048), "standard", 7, 1), ((768, 512), "gram_stabilized", 3, 2), ((300, 700), "gram", 4, 3)]
    assert nsm.muon_ns_workspace_size(7, 1024, 2048) > nsm.NOALLOC_SCRATCH_BYTES
    assert nsm.muon_ns_workspace_size(1, 1024, 2048) <= nsm.NOALLOC_SCRATCH_BYTES
    for shape, mode, count, seed in cases:
        X = [synth.gaussian(*shape, seed=seed * 100 + i, device=DEV, dtype=torch.bfloat16) for i in range(count)]
        ref = [x.clone() for x in X]
        nsm.muon_ns_batched(ref, mode=mode)
        for _ in range(2):
            got = [x.clone() for x in X]
            st = torch.full((count,), -1, dtype=torch.int32, device=DEV)
            nsm.muon_ns_batched_noalloc(got, mode=mode, status=st)
            torch.cuda.synchronize()
            assert st.cpu().tolist() == [0] * count
            for a, b in zip(got, ref):
                assert torch.equal(a, b)


def test_noalloc_rejects_a_matrix_larger_than_its_scratch():
    X = torch.zeros(2048, 7168, device=DEV, dtype=torch.bfloat16)
    assert nsm.muon_ns_workspace_size(1, 2048, 7168) > nsm.NOALLOC_SCRATCH_BYTES
    with pytest.raises(nsm.MuonError):
        nsm.muon_ns_batched_noalloc([X])
