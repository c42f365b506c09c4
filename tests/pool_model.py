"""Slow, list-based model of the segment allocator's stated policy (test reference).

Policy (include/seg_attn.h, "Segment allocator"): appending n tokens to a
sequence first grows its last run in place into the free slots right after it;
the rest goes to the smallest free run that holds all of it (ties: lowest
start), else to the largest free run (ties: highest start), repeatedly.
Release frees every slot of the sequence.  Free runs are maximal runs of free
slots of a plain boolean array."""


class PoolModel:
    def __init__(self, n):
        self.n = n
        self.free = [True] * n
        self.seqs = {}

    def free_runs(self):
        runs, i = [], 0
        while i < self.n:
            if self.free[i]:
                j = i
                while j < self.n and self.free[j]:
                    j += 1
                runs.append((i, j - i))
                i = j
            else:
                i += 1
        return runs

    def _take(self, seq, start, count, out):
        for s in range(start, start + count):
            assert self.free[s]
            self.free[s] = False
            out.append(s)
        runs = self.seqs[seq]
        if runs and runs[-1][0] + runs[-1][1] == start:
            runs[-1] = (runs[-1][0], runs[-1][1] + count)
        else:
            runs.append((start, count))

    def append(self, seq, n):
        if n > sum(self.free):
            return None  # no space, nothing changes
        self.seqs.setdefault(seq, [])
        out, left = [], n
        runs = self.seqs[seq]
        if left and runs:
            end = runs[-1][0] + runs[-1][1]
            k = 0
            while k < left and end + k < self.n and self.free[end + k]:
                k += 1
            if k:
                self._take(seq, end, k, out)
                left -= k
        while left:
            fr = self.free_runs()
            fits = [r for r in fr if r[1] >= left]
            if fits:
                start = min(fits, key=lambda r: (r[1], r[0]))[0]
                take = left
            else:
                start, take = max(fr, key=lambda r: (r[1], r[0]))
            self._take(seq, start, take, out)
            left -= take
        return out

    def release(self, seq):
        for s, l in self.seqs.pop(seq):
            for x in range(s, s + l):
                assert not self.free[x]
                self.free[x] = True

    def stats(self):
        fr = self.free_runs()
        return dict(num_slots=self.n, free_slots=sum(self.free), free_runs=len(fr),
                    largest_free_run=max((l for _, l in fr), default=0),
                    sequences=len(self.seqs), segments=sum(len(v) for v in self.seqs.values()))
