"""The CPU models of the two flash-style kernels' barrier protocols
(test_decode_protocol.py, test_prefill_protocol.py) hard-code the kernels'
buffer counts; these checks read the counts from the CUDA sources so that a
change to a kernel's ring or buffer sizes cannot leave its model silently
checking a different protocol."""
import os
import re

import test_decode_protocol as decode_model
import test_prefill_protocol as prefill_model

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "mla_latent_kv_43_b200", "csrc")


def constants(name):
    text = open(os.path.join(CSRC, name)).read()
    found = {}
    for decl in re.findall(r"constexpr\s+int\s+([^;]+);", text):
        for part in decl.split(","):
            m = re.fullmatch(r"\s*(k\w+)\s*=\s*(\d+)\s*", part)
            if m:
                found[m.group(1)] = int(m.group(2))
    return found


def test_decode_model_matches_the_attention_kernel():
    c = constants("sm100_attend.cu")
    assert c["kStages"] == decode_model.STAGES
    assert c["kXBufs"] == decode_model.XBUFS


def test_prefill_model_matches_the_prefill_kernel():
    c = constants("sm100_prefill.cu")
    assert c["kKStages"] == prefill_model.K_STAGES
    assert c["kVStages"] == prefill_model.V_STAGES
    assert c["kGroups"] == prefill_model.GROUPS
    # four softmax warps per query group: the group's 128 rows are the TMEM lanes
    assert c["kQ"] == 32 * prefill_model.WARPS
