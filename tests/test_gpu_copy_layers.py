"""GPU parity of pa_copy_blocks_layers (one call copies the same block pairs
in every layer's K and V cache) against the oracle's per-layer block copy:
bit-exact, for 1, 3 and 40 layers (the last crosses the 32-layer launch
group) and for more pairs than one launch takes."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_410_b200 import binding as B
from paged_kv_cache_410_b200.session import to_bits

pytestmark = pytest.mark.gpu


def random_pairs(rng, num_blocks, n):
    ids = rng.permutation(num_blocks)[:2 * n]
    return np.stack([ids[:n], ids[n:]], axis=1).astype(np.int32)


@pytest.mark.parametrize("layers,npairs,dtype,bs", [
    (1, 5, "f16", 16), (3, 48, "e4m3", 32), (40, 300, "bf16", 16), (33, 7, "e4m3", 128),
])
def test_matches_per_layer_oracle_copy(layers, npairs, dtype, bs):
    rng = np.random.default_rng(layers * 1000 + npairs)
    nb, hkv, d = 700, 2, 64
    shape = (nb, bs, hkv, d)
    np_t = np.uint8 if dtype == "e4m3" else np.uint16
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8}[dtype]
    host_k = [rng.integers(0, np.iinfo(np_t).max, shape, dtype=np_t) for _ in range(layers)]
    host_v = [rng.integers(0, np.iinfo(np_t).max, shape, dtype=np_t) for _ in range(layers)]
    to_dev = lambda a: (torch.from_numpy(a) if np_t == np.uint8 else
                        torch.from_numpy(a.view(np.int16)).view(tdt)).cuda()
    gk = [to_dev(a) for a in host_k]
    gv = [to_dev(a) for a in host_v]
    pairs = random_pairs(rng, nb, npairs)
    cache = B.PagedCache(nb, bs, hkv, d, tdt)
    B.pa_copy_blocks_layers(pairs, gk, gv, cache)
    torch.cuda.synchronize()
    for layer in range(layers):
        oracle.copy_blocks(pairs, host_k[layer], host_v[layer], dtype)
        assert np.array_equal(to_bits(gk[layer]), host_k[layer]), layer
        assert np.array_equal(to_bits(gv[layer]), host_v[layer]), layer


def test_one_layer_equals_pa_copy_blocks():
    rng = np.random.default_rng(2)
    shape = (300, 16, 8, 128)
    k = torch.randn(shape, device="cuda", dtype=torch.float16)
    v = torch.randn(shape, device="cuda", dtype=torch.float16)
    k2, v2 = k.clone(), v.clone()
    pairs = random_pairs(rng, 300, 40)
    cache = B.PagedCache.for_tensor(k)
    B.pa_copy_blocks(pairs, k, v, cache)
    B.pa_copy_blocks_layers(pairs, [k2], [v2], cache)
    torch.cuda.synchronize()
    assert torch.equal(k, k2) and torch.equal(v, v2)
