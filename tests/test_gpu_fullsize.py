"""Full-size parity: each workload at its full shape (one layer), through the
same entry point and launch configuration the benchmark times
(hkv_encode_keys for the cache, then hkv_decode_step).  Every code, every
selected index and every output row is compared with the oracle."""
import numpy as np
import pytest

import synth
from tests.helpers import margin_inputs
from tests.test_gpu_parity import compare_decode, run_decode

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("name", ["tiny_lsh", "hashevict_lsh", "spotlight_mlp", "signvq", "qwen7b_512k"])
def test_decode_step_full_size(name):
    w = synth.WORKLOADS[name].with_(layers=1) if name == "qwen7b_512k" else synth.WORKLOADS[name]
    inp = margin_inputs(w)
    compare_decode(w, inp, run_decode(w, inp))
