"""The pool pins catch plausible mistakes in the oracle's pool model: each
mutant subclass changes one rule, and at least one pin must fail on it."""
import pytest

from oracle.pool import RULE_SHARED, RefPool
from tests import test_pool as pins


class FreesAtTail(RefPool):
    """Freed blocks appended to the tail instead of prepended (no LIFO reuse)."""
    def _release_refs(self, ordered, counts):
        run = []
        for b in ordered:
            counts[b] -= 1
            if self.ref[b] == 0 and self.pin[b] == 0:
                run.append(b)
        self.free.extend(run)


class ReleasesInOrder(RefPool):
    """A sequence's blocks freed head first instead of in reverse."""
    def release(self, seq_id):
        table = self.tables.pop(seq_id)
        del self.lens[seq_id]
        del self.tail_owned[seq_id]
        self._release_refs(list(table), self.ref)


class CopiesEveryPartialTail(RefPool):
    """Copy-on-write even when the partial tail is not shared."""
    def append(self, seq_id, n):
        t = self.tables[seq_id]
        if t and self.lens[seq_id] % self.block_size and n > 0 and self.ref[t[-1]] == 1:
            self.ref[t[-1]] += 1  # pretend it is shared
            ok = super().append(seq_id, n)
            if not ok:
                self.ref[t[-1]] -= 1
            return ok
        return super().append(seq_id, n)


class NeverCopies(RefPool):
    """Writes into a shared partial tail in place."""
    def append(self, seq_id, n):
        t = self.tables[seq_id]
        if not t:
            return super().append(seq_id, n)
        b, saved = t[-1], self.ref[t[-1]]
        self.ref[b] = 1  # pretend the tail is not shared
        try:
            return super().append(seq_id, n)
        finally:
            self.ref[b] = saved


class OneBlockShort(RefPool):
    """Block count floor(n/B) instead of ceil(n/B)."""
    def append(self, seq_id, n):
        import oracle.pool as op
        real = op.blocks_for
        op.blocks_for = lambda m, b: m // b
        try:
            return super().append(seq_id, n)
        finally:
            op.blocks_for = real


PIN_CALLS = [
    lambda cls, g: pins.test_pagedkv_trace_without_pin(lambda: cls(3, 4), g),
    lambda cls, g: pins.test_one_page_pool_cannot_copy_shared_tail(cls),
    lambda cls, g: pins.test_tail_waste_and_block_counts(cls, g),
    lambda cls, g: pins.test_r7_one_block_appended_and_slot(cls, g),
    lambda cls, g: pins.test_lifo_reuse_and_reverse_free_order(cls),
    lambda cls, g: pins.test_prefix_sharing_refcounts(cls, RULE_SHARED, g),
]


@pytest.mark.parametrize("mutant", [FreesAtTail, ReleasesInOrder, CopiesEveryPartialTail, NeverCopies,
                                    OneBlockShort], ids=lambda c: c.__name__)
def test_pool_pins_catch_mutant(mutant, golden):
    failures = 0
    for call in PIN_CALLS:
        try:
            call(mutant, golden)
        except (AssertionError, Exception):
            failures += 1
    assert failures > 0


def test_pool_pins_pass_on_the_model(golden):
    for call in PIN_CALLS:
        call(RefPool, golden)
