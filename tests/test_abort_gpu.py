"""The kernel's bounded-wait error path, exercised on purpose on the GPU.

Every mbarrier wait in the kernel gives up after a host-set bound; the CTA
then records the site of the first wait that ran out in the device status
word, every role leaves its loop, the producer waits for its own TMA copies,
the MMA issuers wait for their own tensor-core work, and the tensor memory
is freed.  The testing hook makes every softmax warp wait on an mbarrier that
nothing completes; with a 2 ms bound that wait runs out, the whole launch
takes the error path, and afterwards the context must still be usable and a
normal call must be correct.  No fault, trap or endless loop is involved.
"""
import pytest
import torch

import oracle
import seeded_inputs as si
from gpu_helpers import assert_parity, needs_gpu, run_cuda

pytestmark = [pytest.mark.gpu, needs_gpu]

# Device status sites (first timed-out wait): producer 1-3, MMA issuers
# 11-16, softmax 21-22, drains 31, the testing hook's wait 41.  The hook's
# wait normally runs out first; a role that started waiting at about the
# same time may win the race to record its site.
KNOWN_SITES = {1, 2, 3, 11, 12, 13, 14, 15, 16, 21, 22, 31, 41}


@pytest.mark.parametrize("name", ["vit_b16_224px_3views", "siglip_so400m14_224px_2views"])
def test_bounded_wait_runs_out_and_context_recovers(name):
    import vit_self_attention_b200 as vab

    c = si.workload(name)
    bits = c.qkv(0)
    vab.vla_attn_reset_device_status()
    vab.vla_attn_set_wait_limit_ns(2_000_000)
    vab.vla_attn_set_test_stall(True)
    try:
        run_cuda(bits, c.scale)
        st, site = vab.vla_attn_last_device_status()
    finally:
        vab.vla_attn_set_test_stall(False)
        vab.vla_attn_set_wait_limit_ns(0)
        vab.vla_attn_reset_device_status()
    torch.cuda.synchronize()
    assert st == vab.ERR_TIMEOUT, (st, site)
    assert site in KNOWN_SITES, site

    # The context is usable and a normal call gives the right answer.
    got = run_cuda(bits, c.scale)
    assert_parity(got, oracle.attention_packed_bf16(bits, c.scale), f"after abort, {name}")
    st, site = vab.vla_attn_last_device_status()
    assert (st, site) == (0, 0)
