"""Sequential model of the sparse user-id -> dense slot map (test infrastructure only).

Source: "How Generative Recommenders Are Redefining RecSys at Scale", section
"Dynamic embedding" (real user / item ids are sparse, so a hash table maps
them to rows of dense storage); here the dense rows are the KV table's user
slots.  Readings taken:
* slots 0..n_slots-1 are free at first, held on a LIFO stack initialised from
  ``free_order`` (top = last element);
* ``lookup(ids, insert)``: a known id returns its slot; with ``insert`` an
  unknown id takes the slot on top of the stack, ids being served in the order
  listed (a repeated id reuses the slot its first occurrence got); without
  ``insert`` an unknown id returns -1.  A negative id is invalid.  If the stack
  runs out, the call changes nothing and reports OUT_OF_SLOTS;
* ``erase(ids)``: each known id's slot goes back on the stack in the order
  listed; unknown (or already erased) ids are ignored.
"""

from __future__ import annotations

OK, INVALID_ARG, OUT_OF_SLOTS = 0, 1, 2


class UserMapOracle:
    def __init__(self, n_slots, free_order=None):
        order = list(range(n_slots)) if free_order is None else [int(x) for x in free_order]
        assert sorted(order) == list(range(n_slots)), "free order must be a permutation"
        self.stack = order
        self.slot = {}

    def lookup(self, ids, insert):
        ids = [int(i) for i in ids]
        if any(i < 0 for i in ids):
            return INVALID_ARG, [-1] * len(ids)
        stack, slot = list(self.stack), dict(self.slot)
        out = []
        for i in ids:
            if i in slot:
                out.append(slot[i])
            elif insert:
                if not stack:
                    return OUT_OF_SLOTS, [-1] * len(ids)
                slot[i] = stack.pop()
                out.append(slot[i])
            else:
                out.append(-1)
        self.stack, self.slot = stack, slot
        return OK, out

    def erase(self, ids):
        for i in ids:
            s = self.slot.pop(int(i), None)
            if s is not None:
                self.stack.append(s)
        return OK
