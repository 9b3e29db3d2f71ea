"""GPU parity of tree_kv_write against the oracle: bit-exact caches after the
append of the step's tree rows, on ragged geometry (including sequences whose
rows do not fit, which must stay untouched), GQA head counts, both head dims,
the largest tree and several layers."""
import numpy as np
import pytest
import torch

import tree_speculative_decoding_04_b200 as tv
from gpu_helpers import dev

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize(
    "L,B,Hkv,D,M,ks,kl,S_cap",
    [
        (1, 1, 1, 64, 0, [0], [0], 8),  # a single root row at column 0
        (3, 4, 2, 128, 16, [0, 5, 40, 0], [100, 33, 0, 120], 140),  # b3 does not fit
        (2, 3, 8, 128, 255, [0, 0, 7], [1, 300, 44], 560),  # largest tree
        (4, 5, 4, 64, 9, [3, 0, -2, 50, 0], [20, 95, 10, 30, 0], 105),  # negative start, exact fit
    ],
)
def test_parity(orc, L, B, Hkv, D, M, ks, kl, S_cap):
    g = torch.Generator(device=dev()).manual_seed(L * 1000 + M)
    n = M + 1

    def rnd(shape):
        return torch.randint(-32768, 32767, shape, generator=g, device=dev(), dtype=torch.int16).view(torch.bfloat16)

    k = [rnd((B, Hkv, S_cap, D)) for _ in range(L)]
    v = [rnd((B, Hkv, S_cap, D)) for _ in range(L)]
    tk, tvv = rnd((L, B, Hkv, n, D)), rnd((L, B, Hkv, n, D))
    kh, vh = [_u16(t).copy() for t in k], [_u16(t).copy() for t in v]
    ksa, kla = np.asarray(ks, np.int32), np.asarray(kl, np.int32)
    kp, vp = tv.layer_pointers(k), tv.layer_pointers(v)
    tv.tree_kv_write(kp, vp, tk, tvv, S_cap, torch.as_tensor(ksa, device=dev()), torch.as_tensor(kla, device=dev()))
    torch.cuda.synchronize()
    orc.tree_kv_write(kh, vh, _u16(tk), _u16(tvv), ksa, kla)
    for l in range(L):
        np.testing.assert_array_equal(_u16(k[l]), kh[l])
        np.testing.assert_array_equal(_u16(v[l]), vh[l])


def test_rejects_misaligned_rows():
    k = [torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device=dev())]
    kp = tv.layer_pointers(k)
    buf = torch.zeros(2 * 64 + 8, dtype=torch.bfloat16, device=dev())
    tk = buf[1:65].view(1, 1, 1, 1, 64)  # 2-byte offset: not 16-byte aligned
    z = torch.zeros(1, dtype=torch.int32, device=dev())
    with pytest.raises(tv.TVError):
        tv.tree_kv_write(kp, kp, tk, tk, 8, z, z)
