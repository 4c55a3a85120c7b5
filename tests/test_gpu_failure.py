"""Failure detection on the GPU without a GPU fault.

Every wait inside the attention kernel is bounded (about 2 s). A test hook
makes the next launch leave one K tile unloaded in its first work unit, so
the waits that depend on it run out (the MMA issuer's on that tile, or the
producer's on the ring slot that only the stalled MMA would free): the CTA must record the timeout in the
device error word, drain its copies and MMAs, free tensor memory and exit.
The host then reads ATLAS_ERR_TIMEOUT, and the context must stay usable: the
next, normal launch matches the oracle and leaves the error word clear.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from helpers import assert_attn_close, attention_gpu, f64, n_threads, orc
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_expired_wait_reports_timeout_and_context_survives():
    N, L, G, heads, hd = 1536, 768, 300, 2, 128
    mk = lambda n, s: normal((n, heads, hd), s, torch.bfloat16, seed=5, device=DEV)
    q_d, k_d, v_d, q_g, k_g, v_g = (mk(N, "q_d"), mk(N, "k_d"), mk(N, "v_d"),
                                    mk(G, "q_g"), mk(G, "k_g"), mk(G, "v_g"))
    assert atlas.last_device_error() == 0
    atlas.debug_stall_next_attention()
    attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g, with_lse=False)
    torch.cuda.synchronize()                       # the launch returns: no hang
    st = atlas.lib().atlas_last_device_error(None, ctypes.byref(code := ctypes.c_uint32()))
    assert st == atlas.ERR_TIMEOUT
    # The MMA issuer waits on the unloaded tile; the producer, once the ring is
    # full, waits on a slot that only that MMA would free. Both waits start
    # microseconds apart and either may expire first; the other then sees the
    # CTA's abort flag and leaves without a bit of its own.
    assert code.value & 0b11, f"producer/MMA timeout bit missing: 0x{code.value:x}"
    assert not code.value & (1 << 4), f"tensor-memory allocation flagged: 0x{code.value:x}"
    # the word was cleared by the read, and the context still works
    assert atlas.last_device_error() == 0
    o_d, o_g, _ = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g, with_lse=False)
    torch.cuda.synchronize()
    assert atlas.last_device_error() == 0
    ref_d, ref_g, _ = orc().attention_full(f64(q_d), f64(k_d), f64(v_d), L, f64(q_g), f64(k_g),
                                           f64(v_g), 1 / math.sqrt(hd), n_threads())
    assert_attn_close(np.concatenate([f64(o_d), f64(o_g)]), np.concatenate([ref_d, ref_g]),
                      "bf16")
