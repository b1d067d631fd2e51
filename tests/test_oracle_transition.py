"""The block transition of the oracle (CPU): the finished block's K/V join each
sequence's prefix and the next block starts from an empty cache."""
import pins
from oracle import attention, policy, transition


def test_block_transition_pins():
    pins.check_block_transition(transition.grow_prefix, transition.finish_block, transition.next_block_workload,
                                policy.run_policy, attention.attend)
