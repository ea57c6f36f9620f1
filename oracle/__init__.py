"""CPU oracle of the Lighthouse layer: test infrastructure only (see ``oracle.lighthouse``)."""
