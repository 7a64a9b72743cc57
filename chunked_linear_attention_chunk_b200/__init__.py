"""libkda: chunked KDA forward (bounded-decay gated delta rule) for B200 -- placeholder."""
