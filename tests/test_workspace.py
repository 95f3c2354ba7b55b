"""Host-side sizing of the prefill workspace (no GPU needed: nothing is launched).

gdn_chunk_fwd_workspace_size must cover the tensor-core path's layout: a 1 KiB header, per chunk
slot and v-head a 16 KiB [T'; P] tile and 512 B of Gamma and d, then the intra-sequence scan's
fp32 state arrays (one per sequence, three per segment).  The segment length follows the
library's rule from the per-SM share of the chunk work (148 SMs when no GPU can be queried).
"""
import pytest

from gated_deltanet_fwd_b200 import build as gbuild
from gated_deltanet_fwd_b200 import gdn


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gdn.load()


def _sms():
    import torch
    if torch.cuda.is_available():
        return torch.cuda.get_device_properties(0).multi_processor_count
    return 148


def _expected(N, B, T, Hv, sms):
    n_tok = B * T
    slots = -(-n_tok // 64) + N
    per_sm = (-(-n_tok // 64)) * Hv // sms
    chunks = 8
    while chunks * 2 <= per_sm:
        chunks *= 2
    lseg = chunks * 64 if n_tok > 0 else 0
    segs = n_tok // lseg + N if lseg > 0 else 0
    size = 1024 + slots * Hv * (16384 + 512) + (N + 3 * segs) * Hv * 128 * 128 * 4
    return (size + 255) // 256 * 256


CASES = [
    (4, 1, 32768, 16, 32),   # the 32K varlen prefill
    (1, 1, 4096, 16, 32),    # the 4K prefill
    (2, 2, 16384, 16, 32),   # the layer core
    (3, 1, 200, 1, 2),
    (1, 1, 1, 1, 1),
    (5, 5, 0, 2, 4),         # no tokens: header and the per-sequence slots only
]


@pytest.mark.parametrize("case", CASES)
def test_workspace_size_covers_the_layout(lib, case):
    N, B, T, Hk, Hv = case
    got = lib.gdn_chunk_fwd_workspace_size(N, B, T, Hk, Hv, 128, 128, 64)
    assert got == _expected(N, B, T, Hv, _sms())
    assert got % 256 == 0
    # never smaller than the per-chunk operands the fused call requires
    assert got >= 1024 + (-(-(B * T) // 64) + N) * Hv * (16384 + 512)


def test_workspace_size_other_shapes_need_only_the_status_word(lib):
    for dk, dv, chunk in [(64, 64, 64), (128, 128, 32), (128, 64, 64), (16, 16, 16)]:
        assert lib.gdn_chunk_fwd_workspace_size(1, 1, 4096, 1, 2, dk, dv, chunk) == 256


def test_workspace_size_grows_with_tokens(lib):
    sizes = [lib.gdn_chunk_fwd_workspace_size(1, 1, T, 16, 32, 128, 128, 64)
             for T in (64, 128, 1024, 4096, 32768)]
    assert sizes == sorted(sizes) and len(set(sizes)) == len(sizes)
