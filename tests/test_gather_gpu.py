"""GPU page-table copy-out (gqa_paged_gather) is bit-exact against the oracle's copy."""
import numpy as np
import pytest
import torch

from gqa_attention_paged_b200 import binding, inputs
from oracle import oracle
from tests._util import bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gather(kv):
    cu = torch.zeros(len(kv.seq_lens) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(kv.seq_lens.to(torch.int64), 0)
    k, v = binding.gqa_paged_gather(kv.k_pages.to(DEV), kv.v_pages.to(DEV),
                                    kv.page_table.to(DEV), kv.seq_lens.to(DEV), cu.to(DEV),
                                    int(cu[-1]))
    torch.cuda.synchronize()
    return bits(k.cpu()), bits(v.cpu())


@pytest.mark.parametrize("name", ["tiny", "llama7b", "long70b_fp8", "aliased"])
def test_gather_bit_exact(name):
    case = {
        "tiny": lambda: inputs.tiny_decode(seed=0),
        "llama7b": lambda: inputs.llama7b_decode(seed=0),
        "long70b_fp8": lambda: inputs.long70b_decode(seed=0, kv_dtype="fp8_e4m3"),
        "aliased": lambda: inputs.make_decode_case(3, 8, 2, 128, 32, [300, 100, 65], seed=2,
                                                   alias_prefix=[0, 3, 2]),
    }[name]()
    kv = case.kv
    gk, gv = _gather(kv)
    rk, rv = oracle.gather(bits(kv.k_pages), bits(kv.v_pages), kv.page_table.numpy(),
                           kv.seq_lens.numpy())
    assert gk.tobytes() == rk.tobytes()
    assert gv.tobytes() == rv.tobytes()
