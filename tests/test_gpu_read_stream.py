"""pa_read_stream reads every byte once: its XOR fold equals the XOR of the
buffer's 32-bit words computed on the host (bit-exact), for sizes that leave
ragged tails of the grid-stride loop."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("words", [4, 4 * 37, 4 * 148 * 512 * 4 + 12, 4 * 1000003])
def test_read_stream_folds_every_word(words):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_341_b200 import build
    build.ensure_built()
    from paged_kv_cache_341_b200 import pa
    host = np.random.default_rng(words).integers(0, 2**32, size=words, dtype=np.uint64).astype(np.uint32)
    buf = torch.from_numpy(host.view(np.int32)).cuda()
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_read_stream(buf, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host)
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)
